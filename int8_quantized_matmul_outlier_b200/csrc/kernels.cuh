// Launchers for the sm_100a kernels of the decomposed int8 matmul.  Internal
// to libint8mm.so; the public C ABI is include/int8mm.h.
#pragma once

#include <cstdint>
#include <string>
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace i8mm {

// Status bits in the device status word.
constexpr int kStatusTimeout = 1;

// Outliers per chunk of the fp16 product that the prefill GEMM (CTA pairs)
// computes on the tensor cores (kind::f16, K = 16 per step, operand rows of
// 128 bytes); more outliers take more chunks.
constexpr int kOutMma = 64;

// Sets the message returned by int8mm_last_error() on this host thread.
void set_last_error(const std::string& message);

// ---- weight preparation (once per weight) --------------------------------
// Per output column j of W[K,N] (fp16, row-major): absmax over all K rows,
// c_w[j] = 127/absmax, codes rne(w * c_w) clamped to +-127, written in the
// K-blocked, K-major layout Wb[kb][n][0..128) (kb = k / 128, n < N_pad, N_pad
// a multiple of 256; codes past K or N are 0), so that every tensor-core
// operand tile of 128 or 256 rows is one contiguous block of memory.  Wb
// must be zeroed before.  colmax_bits is [N] u32 scratch; it is zeroed here.
constexpr int kWeightRowPad = 256;
cudaError_t launch_weight_prep(const __half* W, int64_t K, int64_t N, uint32_t* colmax_bits, int8_t* Wb,
                               int64_t N_pad, float* c_w, float* inv_cw, int num_sms, cudaStream_t stream);

// ---- activation passes (every forward) -----------------------------------
struct OutlierScratch {
  unsigned long long* colkey;  // [K] (epoch << 16) | max |x| bits; never cleared
  unsigned long long* epoch;   // [1] epoch of the next launch (the last block advances it)
  unsigned* ticket;            // [1] zero between launches
  uint32_t* mask;              // [ceil(K/32)] outlier column bitmask
  int32_t* pre;                // [ceil(K/32)] exclusive prefix of popc over the mask words
  int32_t* idx;                // [K] ascending outlier columns
  int32_t* count;              // [1] |O|
  float* colmax;               // [K] max_i |X[i,j]|
};

// Pass 1: column maxima of X and the outlier set O = {j : colmax_j > alpha}.
// Blocks fold their chunk maxima into colkey with 64-bit atomicMax; keys of
// earlier launches carry a smaller epoch, so colkey needs no clearing.  The
// last block (ticket) writes colmax, mask, pre, idx and count.
cudaError_t launch_outlier_detect(const __half* X, int64_t M, int64_t K, float alpha,
                                  const OutlierScratch& s, cudaStream_t stream);

// Pass 2: per row, absmax over non-outlier columns, c_x = 127/absmax, int8
// codes (outlier columns 0), and the fp16 outlier values scattered as
// X_OT[o][i] = X[i, idx[o]] (o-major, rows ld_xo entries apart).  With
// `pdl`, launched as a programmatic dependent of pass 1: it loads its row of
// X while that pass finishes.
cudaError_t launch_row_quant(const __half* X, int64_t M, int64_t K, const OutlierScratch& s,
                             int8_t* Xq, float* c_x, __half* X_OT, int64_t ld_xo, bool pdl, cudaStream_t stream);

// ---- fused tcgen05 GEMM ---------------------------------------------------
struct GemmArgs {
  int M, N, K;
  int a_row0;              // first row of Xq that this launch computes (M rows from there); the
                           // row pointers below (c_x, X_OT, Y, acc_dump) start at that row
  int N_pad;               // rows per k block in the weight layout
  const float* c_x;        // [M]
  const float* inv_cw;     // [N] 1/c_w (0 where c_w == 0)
  const __half* W;         // [K,N] fp16, rows of the outlier set are read
  const __half* X_OT;      // [|O|][ld_xo] gathered fp16 outlier activations (o-major)
  int ld_xo;               // row stride of X_OT: M rounded up to a multiple of 8
  const int32_t* idx;      // [K] ascending outlier columns
  const int32_t* count;    // [1] |O|
  __half* Y;               // [M,N] fp16 output
  const __half* bias;      // [N] fp16 layer bias added before the rounding, or nullptr
  int32_t* acc_dump;       // [M,N] int32 accumulators, or nullptr
  int split;               // pieces per split tile along K: 1, or 2 .. kGemmMaxTailSplit
  int tail_tiles;          // split > 1: the last tail_tiles tiles are split (the others whole)
  int32_t* sk_ws;          // split > 1: [split-1][tail_tiles][2][128][256] int32 partial tiles
  uint32_t* sk_ticket;     // split > 1: [tail_tiles][2][2] counters, zero between launches
  int* status;             // device status word
  unsigned long long timeout_ns;
  int skip_arrival;        // failure-detection test only: split-K pieces do not count
                           // themselves on the owner's ticket, so its wait runs out
};

// Y = (Xq Wq^T) / (c_x c_w^T) + X[:,O] W[O,:], computed by pairs of CTAs on
// 256 x 256 tiles.  tmA maps Xq [M,K] int8 with 128x128-byte swizzled boxes;
// tmB maps the K-blocked weight Wb as a 2-D array of (K/128 * N_pad) rows of
// 128 bytes with 128-row boxes (the rows of n block j at k block kb start at
// row kb * N_pad + j * kGemmBN).
constexpr int kGemmBM = 128;
constexpr int kGemmBN = 256;
constexpr int kGemmBK = 128;
constexpr int kGemmMaxSplit = 4;      // pieces when every tile is split (also the forced range)
constexpr int kGemmMaxTailSplit = 8;  // pieces when only the leftover tiles are split
// Split K of the CTA-pair GEMM for an M x N x K problem: the last `tail`
// tiles (of the n-major order) are cut into `pieces` along K, the others
// are whole; pieces == 1 is no split.  `force` > 0 cuts every tile into
// that many pieces; 0 picks the plan that best fills the pairs' rounds.
struct GemmSplit {
  int pieces, tail;
};
GemmSplit gemm_split_for(int64_t M, int64_t N, int64_t K, int num_sms, int force);
// With `pdl`, launched as a programmatic dependent of the activation pass:
// its prologue and the first weight-tile loads overlap that pass.
cudaError_t launch_gemm_decomp(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& a, int num_sms,
                               bool pdl, cudaStream_t stream);

// Largest K any kernel here accepts (the row kernels keep a row in registers).
constexpr int64_t kMaxK = 65536;
// Forwards with at most this many rows take the decode GEMM.
constexpr int kDecodeMaxM = 128;

// ---- activation pass in one launch --------------------------------------
// Detection, quantisation and the outlier gather (csrc/xact_rows.cu) for K <=
// kRowActMaxK and at most kRowActMaxRows rows per SM (any M from 1 to 256
// times the SM count; prefill and decode alike): the rows, split into
// equal runs across one block per SM, stream through one shared-memory slot
// per warp and are quantised as they land; a cooperative launch with one
// grid barrier.  Writes idx, count, Xq, c_x and X_OT (not colmax).
struct RowActArgs {
  const __half* X;     // [M, K]
  int M, K;
  int rows_per_block;  // set by the launcher
  int groups;          // set by the launcher: row groups (row slots) per block
  int thr;             // half_magnitude_threshold(alpha)
  int8_t* Xq;          // [M, K]
  float* c_x;          // [M]
  __half* X_OT;        // [|O|][ld_xo]
  int ld_xo;           // row stride of X_OT (M rounded up to a multiple of 8)
  int32_t* idx;        // [K]
  int32_t* count;      // [1]
  uint32_t* omask;     // [2][ceil(K/32)] bitmasks; the one of the current generation is zero
  uint32_t* sync;      // [3] arrivals for generation parity 0 and 1, generation
  int* status;
  unsigned long long timeout_ns;
  int skip_arrival;    // failure-detection test only: block 0 does not arrive at the
                       // grid barrier, so every block's wait there runs out
};
constexpr int64_t kRowActMaxK = 65536;
constexpr int64_t kRowActMaxRows = 256;
constexpr size_t kRowActSmemMax = 220 * 1024;
// Largest binary16 magnitude pattern (0 .. 0x7c00) whose value is <= alpha,
// or -1 when alpha < 0: |x| > alpha exactly when |x|'s bits exceed it.
int half_magnitude_threshold(float alpha);
bool row_act_fits(int64_t M, int64_t K, int num_sms);
cudaError_t launch_row_act(const RowActArgs& a, int num_sms, cudaStream_t stream);

// ---- decode-shape GEMM (M <= 128 tokens) ----------------------------------
struct DecodeArgs {
  int M, N, K;
  int N_pad;               // rows per k block in the weight layout
  const float* c_x;        // [M]
  const float* inv_cw;     // [N]
  const __half* W;         // [K,N] fp16 (outlier rows are read)
  const __half* X_OT;      // [|O|][ld_xo]
  int ld_xo;               // row stride of X_OT (M rounded up to a multiple of 8)
  const int32_t* idx;      // [K]
  const int32_t* count;    // [1]
  __half* Y;               // [M,N]
  const __half* bias;      // [N] or nullptr
  int32_t* acc_dump;       // [M,N] or nullptr
  int32_t* part;           // [kDecodeMaxM][N] int32 partial sums, zero between launches
  unsigned* ticket;        // [ceil(N/128)] k-steps done per n block, zero between launches
  int* status;
  unsigned long long timeout_ns;
  int skip_arrival;        // failure-detection test only: split pieces do not count their
                           // k steps on the owner's ticket, so its wait runs out
  // The activation pass inside the same launch (X != nullptr): the kernel
  // computes O, c_x, Xq, X_OT, idx and count itself and writes them to the
  // buffers below, which c_x, X_OT, idx and count above must name as well.
  const __half* X;         // [M, K] fp16 activations, or nullptr (a separate activation pass ran)
  int thr;                 // half_magnitude_threshold(alpha)
  int8_t* Xq_out;          // [M, K] codes, read back through tmX
  float* c_x_out;          // [M]
  __half* X_OT_out;        // [|O|][ld_xo]
  int32_t* idx_out;        // [K]
  int32_t* count_out;      // [1]
  uint32_t* omask;         // [2][ceil(K/32)] bitmasks by generation parity (as RowActArgs::omask)
  uint32_t* sync;          // [3] arrivals by generation parity, generation (as RowActArgs::sync)
  uint32_t* rowmax;        // [kDecodeMaxM][kRowMaxStride] row absmax bits (first word of
                           // each row), zero between launches
  int skip_barrier;        // failure-detection test only: CTA 0 does not arrive at the first
                           // grid barrier, so every CTA's wait there runs out
};
// Words between the rows of DecodeArgs::rowmax: one 128-byte line per row,
// so that the CTAs' atomics on different rows do not queue on one line.
constexpr int kRowMaxStride = 32;
// Tokens padded to the MMA N of the decode kernel: 16, 32, 64 or 128.
int decode_padded_tokens(int64_t M);
// Whether the decode kernel can run the activation pass itself for M x K
// against N columns: every CTA's slice of X must hold at most 16 vectors of
// 8 columns per row (K <= 16384 on 128 or more SMs).
bool decode_fused_fits(int64_t M, int64_t K, int64_t N, int num_sms);
// tmW maps the K-blocked weight (rows of 128 bytes) with 128-row boxes; tmX
// maps Xq [M,K] with 128 x decode_padded_tokens(M) boxes.  With a.X set, a
// cooperative launch that runs the activation pass too; otherwise, with
// `pdl`, the first weight tiles stream while the activation pass finishes.
cudaError_t launch_gemm_decode(const CUtensorMap& tmW, const CUtensorMap& tmX, const DecodeArgs& a,
                               int num_sms, bool pdl, cudaStream_t stream);

}  // namespace i8mm
