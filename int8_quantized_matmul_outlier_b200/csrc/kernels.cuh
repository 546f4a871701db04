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

// Sets the message returned by int8mm_last_error() on this host thread.
void set_last_error(const std::string& message);

// ---- weight preparation (once per weight) --------------------------------
// Per output column j of W[K,N] (fp16, row-major): absmax over all K rows,
// c_w[j] = 127/absmax, codes rne(w * c_w) clamped to +-127, written
// transposed as Wq_t[N,K] (K-major, the tensor-core operand layout).
// colmax_bits is [N] u32 scratch; it is zeroed here.
cudaError_t launch_weight_prep(const __half* W, int64_t K, int64_t N, uint32_t* colmax_bits,
                               int8_t* Wq_t, float* c_w, float* inv_cw, int num_sms,
                               cudaStream_t stream);

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
// X_OT[o][i] = X[i, idx[o]] (o-major, M entries per o).  With `pdl`,
// launched as a programmatic dependent of pass 1: it loads its row of X
// while that pass finishes.
cudaError_t launch_row_quant(const __half* X, int64_t M, int64_t K, const OutlierScratch& s,
                             int8_t* Xq, float* c_x, __half* X_OT, bool pdl, cudaStream_t stream);

// ---- fused tcgen05 GEMM ---------------------------------------------------
struct GemmArgs {
  int M, N, K;
  const float* c_x;        // [M]
  const float* inv_cw;     // [N] 1/c_w (0 where c_w == 0)
  const __half* W;         // [K,N] fp16, rows of the outlier set are read
  const __half* X_OT;      // [|O|][M] gathered fp16 outlier activations
  const int32_t* idx;      // [K] ascending outlier columns
  const int32_t* count;    // [1] |O|
  __half* Y;               // [M,N] fp16 output
  int32_t* acc_dump;       // [M,N] int32 accumulators, or nullptr
  int* status;             // device status word
  unsigned long long timeout_ns;
};

// Y = (Xq Wq_t^T) / (c_x c_w^T) + X[:,O] W[O,:].  tmA maps Xq [M,K] int8,
// tmB maps Wq_t [N,K] int8, both with 128x128-byte swizzled boxes
// (tmB's box is kGemmBN rows).
constexpr int kGemmBM = 128;
constexpr int kGemmBN = 256;
constexpr int kGemmBK = 128;
// With `pdl`, launched as a programmatic dependent of the row pass: its
// prologue and the first weight-tile loads overlap that pass.
cudaError_t launch_gemm_decomp(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& a,
                               int num_sms, bool pdl, cudaStream_t stream);

}  // namespace i8mm
