// Fused int8 GEMM of the LLM.int8() decomposed matmul for sm_100a.
//
//   Y[i,j] = fp16( Acc[i,j] / (c_x[i] c_w[j]) + sum_{k in O} X[i,k] W[k,j] [+ b[j]] )
//   Acc    = Xq Wq^T, int8 x int8 -> int32 on the 5th-generation tensor cores
//   b      = the layer's optional fp16 bias, added before the one rounding
//
// Method: "LLM.int8() — 大模型激活值里藏着几个超大异常通道", 方法1 (the int8
// product is dequantised by the outer product of the row and column scales)
// and 方法2 (the fp16 product of the outlier columns is added back); the Fig. 2
// caption of the AI 十大核心论文解读 article (Out_i32 dequantised by C_x ⊗ C_w,
// then summed with the fp16 outlier output).  The pages describe this as an
// int8 cuBLAS GEMM followed by a separate fp16 GEMM; here both, and the
// dequantisation, run in one persistent kernel.
//
// Structure: clusters of two CTAs on neighbouring SMs (a CTA pair), one CTA
// per SM, 10 warps each.  A pair computes a 256x256 output tile with
// tcgen05.mma.cta_group::2 (256x256x32 int8) issued by the leader (rank 0);
// each CTA loads its own 128 rows of A and 128 rows of B (TMA completing on
// the leader's barrier), keeps its 128 accumulator rows in its own TMEM and
// writes them; commits reach both CTAs' barriers.  Each SM streams 32 KB per
// 128x256x128 of MMA work through a 6-stage ring.  No TMA multicast is used.
//   warp 0      TMA producer: 128x128 A tiles (Xq) and B tiles (Wq,
//               K-blocked), 128-byte swizzled;
//   warp 1      allocates 512 TMEM columns; in the leader one thread issues
//               tcgen05.mma.kind::i8 into a double-buffered int32
//               accumulator (2 x 256 columns);
//   warps 2-9   epilogue, two warps per TMEM lane quarter (warp w reads lanes
//               32*(w%4)..+31, one output row per thread), each covering one
//               128-column half of the tile: tcgen05.ld of the accumulator,
//               scale by 1/c_x and 1/c_w, write fp16.
// The epilogue of tile t overlaps the main loop of tile t+1.  Every wait is
// bounded; a timeout sets the status word and the CTA drains and exits.
// Problems of at most 128 rows use the same tiles: the peer's 128 rows lie
// past M, where TMA fills zeros and nothing is stored.
//
// The outlier product X[:,O] W[O,:] runs on the tensor cores too, kOutMma
// outliers at a time.  While a tile accumulates, the epilogue warps write the
// first chunk of its operand blocks into shared memory in the
// 128-byte-swizzled K-major layout the int8 tiles use: X_O (this CTA's 128
// rows x the chunk's outliers, from X_OT) and W_O (its 128 columns x those
// outliers, from the rows W[O,:]); both sources are o-major, so each thread
// reads an 8 x 8 block with eight 16-byte loads and transposes it in
// registers.  Once the tile is done they write the dequantised tile back
// into TMEM as fp32; the MMA warp adds X_O W_O^T onto it with
// tcgen05.mma.kind::f16 (K = 16 per step), between the int8 k-blocks of the
// next tile.  With more than kOutMma outliers the epilogue stages the next
// chunk as soon as the tensor cores are done with the blocks, and the MMA
// warp picks it up after its next k-block.  The epilogue then reads the sums.
//
// Split K (when the tiles fill the pairs' rounds badly, e.g. 160 tiles of a
// K-heavy FFN contraction for 74 pairs): every tile is cut into S equal
// ranges of k-blocks, and the S x tiles work units are dealt to the pairs
// piece-major (all first pieces, then all second pieces, ...), so the pairs
// of one round read the same k-slices and keep sharing them in L2.
// The last piece owns the tile.  The other pieces store their exact int32
// partial tiles in a workspace and count themselves on the tile's tickets
// (one per CTA and 128-column half); the owner waits (bounded) for its
// ticket to show the S-1 pieces, adds the partials to its accumulator before
// dequantising, resets the ticket and finishes the tile as an unsplit one.
// A pair deals with all its non-owner units before any owner unit, and
// non-owner units wait on nothing, so every wait ends once all pairs are
// resident (one pair per two SMs; the wait is bounded all the same).
// Integer sums make the result independent of the split.
#include "kernels.cuh"
#include "ptx.cuh"

#include <algorithm>

namespace i8mm {
namespace {

constexpr int BM = kGemmBM, BN = kGemmBN, BK = kGemmBK;
constexpr int A_BYTES = BM * BK;   // 16 KB: 128 rows of A per CTA
constexpr int B_ROWS = BN / 2;     // rows of B per CTA
constexpr int B_BYTES = B_ROWS * BK;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int STAGES = 6;
constexpr int TILE_M = 2 * BM;     // rows per tile
constexpr int NUM_EPI_WARPS = 8;
constexpr int HALF_N = BN / 2;
// The outlier product of tile t is issued after this many int8 k-blocks of
// tile t+1 (by then the epilogue has written tile t back to TMEM), splitting
// the k-block loop in two tight loops.
constexpr int OUT_ISSUE_KB = 16;
constexpr int TMEM_COLS = 2 * BN;
constexpr int NUM_THREADS = 64 + 32 * NUM_EPI_WARPS;
static_assert(TMEM_COLS == 512, "two 128x256 int32 accumulators fill TMEM");

// Shared memory: the ring of 6 stages (A 16 KB + B 16 KB), the barriers:
// full, empty, tmem_full[2], tmem_empty[2], drain, and for the outlier
// product: tile dequantised (operands staged)[2], product done[2]; then the
// outlier product's operand blocks (128 rows of 128 bytes each: up to 64
// fp16 outliers for 128 rows of X_O, and for 128 columns of W_O) and 1/c_w of
// the tile's columns.
constexpr int BAR_OFFSET = STAGES * STAGE_BYTES;
constexpr int NUM_BARS = 2 * STAGES + 5 + 4;
constexpr int MISC_OFFSET = BAR_OFFSET + NUM_BARS * 8;
constexpr int OA_OFFSET = (MISC_OFFSET + 16 + 1023) & ~1023;
constexpr int OB_OFFSET = OA_OFFSET + A_BYTES;
constexpr int RW_OFFSET = OB_OFFSET + A_BYTES;
constexpr int RW_BYTES = 2 * HALF_N * 4;
constexpr int SMEM_BYTES = RW_OFFSET + RW_BYTES + 1024;  // + slack to align the base to 1024
constexpr uint32_t IDESC_F16 = idesc_f16_f32(TILE_M, BN);
constexpr uint32_t IDESC = idesc_i8(TILE_M, BN);
static_assert(SMEM_BYTES <= 232448, "fits the 227 KB of shared memory per block");
static_assert(STAGE_BYTES % 1024 == 0, "stages stay 1024-byte aligned for the 128B swizzle");
static_assert(kOutMma == 64, "a chunk of outliers fills one 128-byte operand row");

__device__ __forceinline__ void fail(const GemmArgs& a, volatile int* abort_flag) {
  *abort_flag = 1;
  atomicOr(a.status, kStatusTimeout);
}

// Wait until the kernel this one depends on (programmatic dependent launch)
// has finished and its memory is visible; a no-op without that launch mode.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// A named barrier over nthreads threads that also returns whether v holds
// on all of them.
__device__ __forceinline__ bool named_bar_and(uint32_t id, uint32_t nthreads, bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 q, %1, 0;\n bar.red.and.pred p, %2, %3, q;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ float dequant(uint32_t acc, float rx, float rw) {
  return __fmul_rn(__fmul_rn(__int2float_rn(static_cast<int>(acc)), rx), rw);
}

// The layer bias of 32 columns n.. (16 when only those are inside N), as
// fp32; zero without a bias.  The same addresses for every lane of the warp.
__device__ __forceinline__ void load_bias32(const __half* bias, int n, bool full32, float (&b)[32]) {
#pragma unroll
  for (int i = 0; i < 32; ++i) b[i] = 0.0f;
  if (bias == nullptr) return;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    if (c < 2 || full32) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(bias + n) + c);
      const __half2* h2 = reinterpret_cast<const __half2*>(&u);
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const float2 f = __half22float2(h2[p]);
        b[8 * c + 2 * p] = f.x;
        b[8 * c + 2 * p + 1] = f.y;
      }
    }
  }
}

// One work unit: k-blocks [kb0, kb1) of a tile cut into S pieces; piece S-1
// finishes the tile.  With split K the last `tail` tiles are the split ones
// (ti: a split tile's index among them); the others are whole units.
struct Unit {
  int tile, piece, S, ti, kb0, kb1;
};

template <bool SPLIT>
__device__ __forceinline__ Unit unit_at(int u, int num_tiles, int num_kb, int tail, int split) {
  const int n_whole = num_tiles - tail;
  if (!SPLIT || u < n_whole) return Unit{u, 0, 1, 0, 0, num_kb};
  Unit w;
  const int t = u - n_whole;
  w.piece = t / tail;
  w.ti = t - w.piece * tail;
  w.tile = n_whole + w.ti;
  w.S = split;
  w.kb0 = w.piece * num_kb / split;
  w.kb1 = (w.piece + 1) * num_kb / split;
  return w;
}

// BIAS: the layer bias is added; SPLIT: split K.  Separate instantiations,
// so that the common path carries none of their code.
template <bool BIAS, bool SPLIT>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_i8_decomp_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                          const GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + BAR_OFFSET);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* tdeq = drain + 1;  // [2] operands staged and tile dequantised into TMEM (leader)
  uint64_t* tout = tdeq + 2;   // [2] outlier product added
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + MISC_OFFSET);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + MISC_OFFSET + 4);
  volatile int* part_ok = reinterpret_cast<volatile int*>(smem + MISC_OFFSET + 8);  // [2] per half

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int M = a.M, N = a.N, K = a.K;
  // a pair of CTAs (a cluster of 2) shares each tile; rank 0 issues the MMAs
  const uint32_t rank = cluster_ctarank();
  const int tile0 = static_cast<int>(blockIdx.x) / 2;
  const int tstride = static_cast<int>(gridDim.x) / 2;
  const int num_m = (M + TILE_M - 1) / TILE_M;
  const int num_n = (N + BN - 1) / BN;
  const int num_tiles = num_m * num_n;
  const int num_kb = (K + BK - 1) / BK;
  const int S = SPLIT ? a.split : 1;        // pieces per split tile
  const int tail = SPLIT ? a.tail_tiles : 0;  // the last `tail` tiles are split
  const int num_units = num_tiles - tail + tail * S;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], NUM_EPI_WARPS * 2);
    }
    mbar_init(drain, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tdeq[b], NUM_EPI_WARPS * 2);
      mbar_init(&tout[b], 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // the peer's barriers are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const unsigned long long tmo = a.timeout_ns;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_phase = 0;
      bool ok = true;
      // Both CTAs' loads complete on the leader's full barrier, and the
      // leader alone announces the pair's bytes.
      auto full_of = [&](int st) { return mapa_shared(smem_u32(&full[st]), 0); };
      // Xq is read again by every column tile of its rows: keep it in L2 ahead
      // of the weight and Y, which stream through once (175B prefill: 843 ->
      // 747 MB of DRAM reads per launch, same time)
      const uint64_t pol_a = l2_policy_evict_last();
      auto expect = [&](int st) {
        if (rank == 0) mbar_arrive_expect_tx(&full[st], 2 * STAGE_BYTES);
      };
      auto load_a = [&](int st, int kb, int m_blk) {
        const int row = a.a_row0 + m_blk * TILE_M + static_cast<int>(rank) * BM;
        tma_load_2d_pair_hint(smem + st * STAGE_BYTES, &tmA, full_of(st), kb * BK, row, pol_a);
      };
      auto load_b = [&](int st, int kb, int n_blk) {
        const int row = kb * a.N_pad + n_blk * BN + static_cast<int>(rank) * B_ROWS;
        tma_load_2d_pair(smem + st * STAGE_BYTES + A_BYTES, &tmB, full_of(st), 0, row);
      };
      // The weight tiles of the first k-blocks do not depend on the
      // activation pass: issue them before waiting for it, then the
      // matching activation tiles (all stages start empty).
      const Unit first = unit_at<SPLIT>(tile0, num_tiles, num_kb, tail, S);
      const int pre = tile0 < num_units ? min(STAGES, first.kb1 - first.kb0) : 0;
      for (int i = 0; i < pre; ++i) {
        expect(i);
        load_b(i, first.kb0 + i, first.tile / num_m);
      }
      pdl_wait();
      for (int i = 0; i < pre; ++i) {
        load_a(i, first.kb0 + i, first.tile % num_m);
        issued_mask |= 1u << i;
      }
      stage = pre % STAGES;
      phase = pre == STAGES ? 1u : 0u;
      for (int u = tile0; u < num_units && ok; u += tstride) {
        const Unit w = unit_at<SPLIT>(u, num_tiles, num_kb, tail, S);
        const int m_blk = w.tile % num_m, n_blk = w.tile / num_m;
        for (int kb = w.kb0 + (u == tile0 ? pre : 0); kb < w.kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, tmo, abort_flag)) {
            ok = false;
            break;
          }
          expect(stage);
          load_a(stage, kb, m_blk);
          load_b(stage, kb, n_blk);
          issued_mask |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        fail(a, abort_flag);
        // Let every load already issued land before the CTA can exit (the
        // peer cannot watch the leader's barriers: it waits a while).
        if (rank == 0) {
          for (int s = 0; s < STAGES; ++s)
            if (issued_mask & (1u << s)) mbar_wait(&full[s], (issued_phase >> s) & 1u, tmo, nullptr);
        } else {
          const uint64_t t0 = global_timer_ns();
          while (global_timer_ns() - t0 < 200000ull) {
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // -------------------------------------------------------- MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int lt = 0;
      // Outlier product of a finished tile: once the epilogue has staged a
      // chunk of operand blocks (and, for the first, written the dequantised
      // tile back to TMEM), D += X_O W_O^T in up to 64/16 steps of K = 16;
      // the first chunk after OUT_ISSUE_KB int8 k-blocks of the next tile.
      pdl_wait();
      const int cnt = *a.count;
      const int nchunks = (cnt + kOutMma - 1) / kOutMma;
      // tdeq/tout phases used so far per accumulator buffer: one per chunk of
      // every tile whose product ran there (with split K only units that
      // finish a tile have one)
      uint32_t chunk_ph[2] = {0u, 0u};
      int pend = -1;        // accumulator buffer whose outlier product is due
      int pend_chunk = 0;   // its next chunk
      uint32_t pend_base = 0;
      // Issues the next chunk of the pending product once the epilogue has
      // staged it.  `block`: wait for that (bounded); otherwise only look.
      // Returns 1 when issued, 0 when not ready yet, -1 after a timeout.
      auto issue_chunk = [&](bool block) -> int {
        const uint32_t par = (pend_base + static_cast<uint32_t>(pend_chunk)) & 1u;
        if (block) {
          if (!mbar_wait(&tdeq[pend], par, tmo, abort_flag)) return -1;
        } else if (!mbar_try_wait(&tdeq[pend], par)) {
          return 0;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(pend * BN);
        const uint64_t adesc = smem_desc_k_sw128(smem_u32(smem + OA_OFFSET));
        const uint64_t bdesc = smem_desc_k_sw128(smem_u32(smem + OB_OFFSET));
        const int nk = (min(cnt - pend_chunk * kOutMma, kOutMma) + 15) / 16;
        for (int kk = 0; kk < nk; ++kk)  // 32 bytes (16 fp16) along K per step
          mma_f16_pair(d_tmem, adesc + static_cast<uint64_t>(kk * 2), bdesc + static_cast<uint64_t>(kk * 2),
                       IDESC_F16, 1u);
        mma_commit_pair(&tout[pend], 0x3);
        if (++pend_chunk == nchunks) pend = -1;
        return 1;
      };
      for (int u = tile0; u < num_units && ok; u += tstride, ++lt) {
        const Unit w = unit_at<SPLIT>(u, num_tiles, num_kb, tail, S);
        const int buf = lt & 1;
        const uint32_t use = static_cast<uint32_t>(lt >> 1);
        if (!mbar_wait(&tempty[buf], (use & 1u) ^ 1u, tmo, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
        auto kblock = [&](int kb) -> bool {
          if (!mbar_wait(&full[stage], phase, tmo, abort_flag)) return false;
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
          const uint64_t adesc = smem_desc_k_sw128(sa);
          const uint64_t bdesc = smem_desc_k_sw128(sa + A_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk)  // advance 32 bytes along K inside the 128-byte swizzled row
            mma_i8_pair(d_tmem, adesc + static_cast<uint64_t>(kk * 2), bdesc + static_cast<uint64_t>(kk * 2), IDESC,
                        (kb != w.kb0 || kk != 0) ? 1u : 0u);
          mma_commit_pair(&empty[stage], 0x3);  // frees the stage in both CTAs
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
          return true;
        };
        const int ksplit = pend >= 0 ? min(w.kb1, w.kb0 + OUT_ISSUE_KB) : w.kb1;
        int kb = w.kb0;
        for (; kb < ksplit && ok; ++kb) ok = kblock(kb);
        if (ok && pend >= 0) ok = issue_chunk(true) > 0;
        // more than kOutMma outliers: the later chunks go in as soon as the
        // epilogue has staged them, looked for after every k-block
        for (; kb < w.kb1 && ok && pend >= 0; ++kb) {
          ok = kblock(kb);
          if (ok) ok = issue_chunk(false) >= 0;
        }
        for (; kb < w.kb1 && ok; ++kb) ok = kblock(kb);
        if (ok) mma_commit_pair(&tfull[buf], 0x3);
        // the previous tile's product is complete before this one's is due
        while (ok && pend >= 0) ok = issue_chunk(true) > 0;
        if (nchunks > 0 && w.piece == w.S - 1) {  // the tile is complete: its outlier product is due
          pend = buf;
          pend_chunk = 0;
          pend_base = chunk_ph[buf];
          chunk_ph[buf] += static_cast<uint32_t>(nchunks);
        }
      }
      while (ok && pend >= 0) ok = issue_chunk(true) > 0;
      if (!ok) {
        fail(a, abort_flag);
        mma_commit_pair(drain, 0x1);
        mbar_wait(drain, 0, tmo, nullptr);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;                  // 0..7
    const int q = warp & 3;                   // TMEM lane quarter this warp may read
    const int h = ew >> 2;                    // 128-column half of the tile
    const int tl = (ew & 3) * 32 + lane;      // thread index among the half's 4 warps
    const int row_t = q * 32 + lane;
    pdl_wait();  // count, idx, X_OT and c_x come from the activation pass
    const int cnt = *a.count;
    const int nchunks = (cnt + kOutMma - 1) / kOutMma;
    float* rws = reinterpret_cast<float*>(smem + RW_OFFSET) + h * HALF_N;  // [HALF_N]
    const uint32_t bar_id = 1 + h;
    const bool y32 = (reinterpret_cast<uintptr_t>(a.Y) & 31u) == 0;
    bool alive = true;
    int lt = 0;
    uint32_t chunk_ph[2] = {0u, 0u};  // tdeq/tout phases used per accumulator buffer (one per chunk)
    // Stages this thread's share of the operand blocks for outliers
    // [64 c, 64 c + 64) of tile (m_blk, n_blk): half 0 writes X_O (rows m of
    // this CTA x outliers, from X_OT[o][m]), half 1 W_O (columns n x
    // outliers, from W[O_o][n]).  Thread tl takes the 8 x 8 block of rows
    // 8 (tl >> 3) .. +7 and outliers 8 (tl & 7) .. +7: eight 16-byte loads
    // along the rows, transposed in registers into eight 16-byte pieces of
    // the 128-byte-swizzled K-major layout (piece j of row r stored at piece
    // j ^ (r % 8), groups of 8 rows 1024 bytes apart).  Only the outliers the
    // product reads (whole K = 16 steps) are written; zero past |O| and
    // past M or N.
    auto stage_chunk = [&](int c, int m_blk, int n_blk) {
      const int o0 = c * kOutMma;
      const int no = min(cnt - o0, kOutMma);
      const int og = tl & 7, rg = tl >> 3;  // outlier group, row group
      if (og >= 2 * ((no + 15) / 16)) return;  // not read by the product
      const int r0 = (h == 0 ? m_blk * TILE_M + static_cast<int>(rank) * BM
                             : n_blk * BN + static_cast<int>(rank) * B_ROWS) + 8 * rg;
      const int lim = h == 0 ? M : N;
      uint4 v[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int o = 8 * og + r;
        v[r] = make_uint4(0u, 0u, 0u, 0u);
        if (o < no && r0 < lim) {
          const __half* src = h == 0 ? a.X_OT + static_cast<size_t>(o0 + o) * a.ld_xo + r0
                                     : a.W + static_cast<size_t>(__ldg(a.idx + o0 + o)) * N + r0;
          v[r] = __ldg(reinterpret_cast<const uint4*>(src));
        }
      }
      if (r0 + 8 > lim) {  // rows past M in the last group of X_O: zero them
        const int keep = max(0, lim - r0);
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          uint32_t* wv = &v[r].x;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            if (2 * e >= keep) wv[e] = 0u;
            else if (2 * e + 1 >= keep) wv[e] &= 0xffffu;
          }
        }
      }
      uint4 t[8];
      transpose8x8_b16(v, t);
      uint8_t* blk = smem + (h == 0 ? OA_OFFSET : OB_OFFSET) + rg * 1024;
#pragma unroll
      for (int i = 0; i < 8; ++i)  // row 8 rg + i of the block, outliers 8 og ..
        *reinterpret_cast<uint4*>(blk + i * 128 + ((og ^ i) << 4)) = t[i];
    };
    // makes this warp's staged pieces visible to the tensor cores and
    // counts it on the leader's tdeq barrier
    auto hand_over = [&](int buf) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tdeq[buf]), 0));
    };
    for (int u = tile0; u < num_units; u += tstride, ++lt) {
      const Unit w = unit_at<SPLIT>(u, num_tiles, num_kb, tail, S);
      const int tile = w.tile;
      const int m_blk = tile % num_m, n_blk = tile / num_m;
      // a unit that finishes its tile (always, without split K); the others
      // only hand their partial sums on
      const bool fin = w.piece == w.S - 1;
      const bool outl_u = cnt > 0 && fin;
      const int buf = lt & 1;
      const uint32_t use = static_cast<uint32_t>(lt >> 1);
      const uint32_t cbase = chunk_ph[buf];  // phase of this tile's first chunk
      if (outl_u) chunk_ph[buf] += static_cast<uint32_t>(nchunks);
      const int nh = n_blk * BN + h * HALF_N;  // first column of this half
      const int m = m_blk * TILE_M + static_cast<int>(rank) * BM + row_t;
      const bool row_ok = m < M;

      // (1) stage this tile's column scales and the first chunk of its
      //     outlier-product operands while the tensor cores still accumulate
      //     the tile (the previous tile's product has completed, waited for
      //     below, so the blocks are free)
      named_bar_sync(bar_id, 128);  // readers of the previous tile are done
      if (fin && tl < HALF_N / 4) {
        const int n = nh + tl * 4;
        const float4 f = n < N ? __ldg(reinterpret_cast<const float4*>(a.inv_cw + n)) : make_float4(0.f, 0.f, 0.f, 0.f);
        reinterpret_cast<float4*>(rws)[tl] = f;
      }
      if (outl_u) stage_chunk(0, m_blk, n_blk);
      float rx = 0.0f;
      if (row_ok) {
        const float c = a.c_x[m];
        rx = c == 0.0f ? 0.0f : __frcp_rn(c);
      }
      if (SPLIT && fin && h == 0 && tl == 0) {
        // the other pieces' partial tiles (normally stored long before): pull
        // them into L2 while the tensor cores finish this piece
        for (int p = 0; p < w.S - 1; ++p)
          bulk_prefetch_l2(a.sk_ws + ((static_cast<size_t>(p) * tail + w.ti) * 2 + rank) * (BM * BN),
                           BM * BN * 4);
      }
      named_bar_sync(bar_id, 128);  // staging visible to the half's 4 warps

      // (2) wait for the accumulator (all lanes; the vote keeps the warp
      //     converged for tcgen05.ld).  After a timeout the warp keeps taking
      //     part in the named barriers but does no more work.
      if (alive) {
        alive = __all_sync(0xffffffffu, mbar_wait(&tfull[buf], use & 1u, tmo, abort_flag));
        if (!alive && lane == 0) fail(a, abort_flag);
      }
      // with split K more named barriers follow: the half's warps decide together
      if (SPLIT) alive = named_bar_and(bar_id, 128, alive);
      if (!alive) continue;
      tc_fence_after();
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(buf * BN + h * HALF_N);
      // piece p's partial sums of this thread's 32-column chunk ch, as 8
      // int4: the workspace holds [piece][tile][CTA rank][half][chunk][int4
      // t4][row] so that a warp's access is 512 contiguous bytes
      auto part_at = [&](int p, int ch) {
        return reinterpret_cast<int4*>(a.sk_ws + ((static_cast<size_t>(p) * tail + w.ti) * 2 + rank) * (BM * BN)) +
               (h * (HALF_N / 32) + ch) * 8 * BM + row_t;
      };
      uint32_t* ticket = SPLIT ? a.sk_ticket + (static_cast<size_t>(w.ti) * 2 + rank) * 2 + h : nullptr;
      if (SPLIT && !fin) {
        // a piece that does not finish the tile: store the partial sums,
        // then count this half on the owner's ticket
#pragma unroll 1
        for (int ch = 0; ch < HALF_N / 32; ++ch) {
          const int cl = ch * 32;
          uint32_t r[32];
          tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(cl), r);
          tmem_wait_ld();
          if (ch == HALF_N / 32 - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[buf]), 0));
          }
          int4* pp = part_at(w.piece, ch);
#pragma unroll
          for (int t4 = 0; t4 < 8; ++t4)
            pp[t4 * BM] = make_int4(static_cast<int>(r[4 * t4]), static_cast<int>(r[4 * t4 + 1]),
                                    static_cast<int>(r[4 * t4 + 2]), static_cast<int>(r[4 * t4 + 3]));
        }
        __threadfence();
        named_bar_sync(bar_id, 128);
        if (tl == 0 && !a.skip_arrival) red_release_add_gpu(ticket, 1u);
        continue;
      }
      if (SPLIT && w.S > 1) {
        // the owner: wait until the other S-1 pieces of this half are stored
        if (tl == 0) {
          const uint32_t need = static_cast<uint32_t>(w.S - 1);
          int got = 1;
          if (ld_acquire_gpu_u32(ticket) != need) {
            const uint64_t t0 = global_timer_ns();
            for (uint32_t it = 1; ld_acquire_gpu_u32(ticket) != need; ++it) {
              if ((it & 15u) == 0 && (*abort_flag || global_timer_ns() - t0 > tmo)) {
                got = 0;
                break;
              }
            }
          }
          if (got) *ticket = 0u;  // ready for the next launch
          else fail(a, abort_flag);
          part_ok[h] = got;
        }
        named_bar_sync(bar_id, 128);
        if (!part_ok[h]) {  // the next unit's first barrier orders the reuse of part_ok
          alive = false;
          continue;
        }
      }
      // adds the other pieces' partial sums to the 32 accumulator columns of chunk ch
      auto add_parts = [&](uint32_t(&r)[32], int ch) {
        for (int p = 0; p < w.S - 1; ++p) {
          const int4* pp = part_at(p, ch);
          int4 v[8];
#pragma unroll
          for (int t4 = 0; t4 < 8; ++t4) v[t4] = __ldcg(pp + t4 * BM);
#pragma unroll
          for (int t4 = 0; t4 < 8; ++t4) {
            r[4 * t4 + 0] += static_cast<uint32_t>(v[t4].x);
            r[4 * t4 + 1] += static_cast<uint32_t>(v[t4].y);
            r[4 * t4 + 2] += static_cast<uint32_t>(v[t4].z);
            r[4 * t4 + 3] += static_cast<uint32_t>(v[t4].w);
          }
        }
      };
      if (outl_u) {
        // (3) dequantise in place (int32 -> fp32 in TMEM), hand the tile to
        //     the MMA warp for the outlier product, chunk by chunk, and wait
        //     for it
#pragma unroll 1
        for (int ch = 0; ch < HALF_N / 32; ++ch) {
          const int cl = ch * 32;
          uint32_t r[32];
          tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(cl), r);
          tmem_wait_ld();
          if (SPLIT) add_parts(r, ch);
          const int n = nh + cl;
          if (a.acc_dump != nullptr && row_ok && n < N) {
            uint4* ap = reinterpret_cast<uint4*>(a.acc_dump + static_cast<size_t>(m) * N + n);
#pragma unroll
            for (int t4 = 0; t4 < 8; ++t4)
              if (n + 32 <= N || t4 < 4) ap[t4] = make_uint4(r[4 * t4], r[4 * t4 + 1], r[4 * t4 + 2], r[4 * t4 + 3]);
          }
          const float4* rw4 = reinterpret_cast<const float4*>(rws + cl);
          if (BIAS) {
            float bb[32];
            load_bias32(n < N ? a.bias : nullptr, n, n + 32 <= N, bb);
#pragma unroll
            for (int t4 = 0; t4 < 8; ++t4) {
              const float4 w = rw4[t4];
              r[4 * t4 + 0] = __float_as_uint(__fadd_rn(dequant(r[4 * t4 + 0], rx, w.x), bb[4 * t4 + 0]));
              r[4 * t4 + 1] = __float_as_uint(__fadd_rn(dequant(r[4 * t4 + 1], rx, w.y), bb[4 * t4 + 1]));
              r[4 * t4 + 2] = __float_as_uint(__fadd_rn(dequant(r[4 * t4 + 2], rx, w.z), bb[4 * t4 + 2]));
              r[4 * t4 + 3] = __float_as_uint(__fadd_rn(dequant(r[4 * t4 + 3], rx, w.w), bb[4 * t4 + 3]));
            }
          } else {
#pragma unroll
            for (int t4 = 0; t4 < 8; ++t4) {
              const float4 w = rw4[t4];
              r[4 * t4 + 0] = __float_as_uint(dequant(r[4 * t4 + 0], rx, w.x));
              r[4 * t4 + 1] = __float_as_uint(dequant(r[4 * t4 + 1], rx, w.y));
              r[4 * t4 + 2] = __float_as_uint(dequant(r[4 * t4 + 2], rx, w.z));
              r[4 * t4 + 3] = __float_as_uint(dequant(r[4 * t4 + 3], rx, w.w));
            }
          }
          tmem_st_32x32b_x32(t_row + static_cast<uint32_t>(cl), r);
        }
        tmem_wait_st();
        tc_fence_before();
        hand_over(buf);
        // the other chunks: once the tensor cores are done with a chunk's
        // operand blocks, stage the next one there and hand it over
        for (int c = 1; c < nchunks && alive; ++c) {
          alive = __all_sync(0xffffffffu, mbar_wait(&tout[buf], (cbase + c - 1) & 1u, tmo, abort_flag));
          if (!alive) break;
          stage_chunk(c, m_blk, n_blk);
          hand_over(buf);
        }
        if (alive) alive = __all_sync(0xffffffffu, mbar_wait(&tout[buf], (cbase + nchunks - 1) & 1u, tmo, abort_flag));
        if (!alive) {
          if (lane == 0) fail(a, abort_flag);
          continue;
        }
        tc_fence_after();
      }
#pragma unroll 1
      for (int ch = 0; ch < HALF_N / 32; ++ch) {
        const int cl = ch * 32;
        uint32_t r[32];
        tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(cl), r);
        tmem_wait_ld();
        if (ch == HALF_N / 32 - 1) {  // accumulator buffer no longer read: release it (the leader's barrier)
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[buf]), 0));
        }
        const int n = nh + cl;
        if (n >= N) continue;  // warp-uniform
        if (SPLIT && !outl_u) add_parts(r, ch);
        const bool full32 = n + 32 <= N;
        float v[32];
        if (outl_u) {  // already dequantised, outlier product included
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
        } else {
          const float4* rw4 = reinterpret_cast<const float4*>(rws + cl);
#pragma unroll
          for (int t4 = 0; t4 < 8; ++t4) {
            const float4 w = rw4[t4];
            v[4 * t4 + 0] = dequant(r[4 * t4 + 0], rx, w.x);
            v[4 * t4 + 1] = dequant(r[4 * t4 + 1], rx, w.y);
            v[4 * t4 + 2] = dequant(r[4 * t4 + 2], rx, w.z);
            v[4 * t4 + 3] = dequant(r[4 * t4 + 3], rx, w.w);
          }
          if (BIAS) {
            float bb[32];
            load_bias32(a.bias, n, full32, bb);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __fadd_rn(v[i], bb[i]);
          }
        }
        if (row_ok) {
          uint4* yp = reinterpret_cast<uint4*>(a.Y + static_cast<size_t>(m) * N + n);
          uint4 out[4];
          uint32_t* ou = reinterpret_cast<uint32_t*>(out);
#pragma unroll
          for (int p = 0; p < 16; ++p) {
            const __half2 hh = __floats2half2_rn(v[2 * p], v[2 * p + 1]);
            ou[p] = *reinterpret_cast<const uint32_t*>(&hh);
          }
          if (y32) {  // whole 32-byte sectors per store
            st_global_256(yp, out[0], out[1]);
            if (full32) st_global_256(yp + 2, out[2], out[3]);
          } else {
            yp[0] = out[0];
            yp[1] = out[1];
            if (full32) {
              yp[2] = out[2];
              yp[3] = out[3];
            }
          }
          if (a.acc_dump != nullptr && !outl_u) {
            uint4* ap = reinterpret_cast<uint4*>(a.acc_dump + static_cast<size_t>(m) * N + n);
#pragma unroll
            for (int t4 = 0; t4 < 8; ++t4)
              if (full32 || t4 < 4) ap[t4] = make_uint4(r[4 * t4], r[4 * t4 + 1], r[4 * t4 + 2], r[4 * t4 + 3]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no CTA leaves while its peer may still signal it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

template <bool BIAS, bool SPLIT>
cudaError_t launch_t(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& a, int num_sms, bool pdl,
                     cudaStream_t stream) {
  auto kern = gemm_i8_decomp_kernel<BIAS, SPLIT>;
  static unsigned long long attr_set = 0;  // one bit per device
  int dev = 0;
  cudaGetDevice(&dev);
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_set & bit)) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set |= bit;
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attrs[2];
  int n = 0;
  attrs[n].id = cudaLaunchAttributeClusterDimension;
  attrs[n].val.clusterDim.x = 2;
  attrs[n].val.clusterDim.y = 1;
  attrs[n].val.clusterDim.z = 1;
  ++n;
  if (pdl) {
    attrs[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  const int num_tiles = ((a.M + TILE_M - 1) / TILE_M) * ((a.N + BN - 1) / BN);
  const int units_of_work = SPLIT ? num_tiles - a.tail_tiles + a.tail_tiles * a.split : num_tiles;
  // one CTA pair per pair of SMs, all resident at once: owners of split
  // tiles wait on other pairs' pieces
  const int slots = num_sms / 2;
  cfg.gridDim = dim3(std::max(1, std::min(units_of_work, slots)) * 2);
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = stream;
  cfg.attrs = attrs;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, tmA, tmB, a);
}

}  // namespace

GemmSplit gemm_split_for(int64_t M, int64_t N, int64_t K, int num_sms, int force) {
  const int64_t tiles = ((M + TILE_M - 1) / TILE_M) * ((N + BN - 1) / BN);
  const int64_t pairs = std::max(1, num_sms / 2);
  const int64_t num_kb = (K + BK - 1) / BK;
  if (force > 0) {  // every tile in `force` pieces
    const int s = static_cast<int>(std::min<int64_t>(force, num_kb));
    return GemmSplit{s, s > 1 ? static_cast<int>(tiles) : 0};
  }
  // Time of the slowest pair, in k-blocks: rounds of units x (k-blocks per
  // unit + a fixed cost per unit of about 16 k-blocks, as measured on a
  // 2048 x 20480 x 5120 contraction: the pipeline turn-around and the
  // owner's pass over the partial tiles).  Candidates: every tile cut into
  // s pieces, or only the tiles past the last full round of pairs (the
  // whole rounds then run unsplit and the leftover tiles are spread over
  // all pairs) in pieces of at least 24 k-blocks (shorter ones measured
  // slower than the model says: 768 x 5120 x 20480 took 75.6 us in pieces of
  // 10 k-blocks and 73.6 us in pieces of 20, against 69.7 us unsplit; the
  // contraction's 26.7 k-block pieces gain 8%).
  auto cost = [&](int64_t whole, int64_t split_tiles, int64_t s) {
    const int64_t whole_rounds = (whole + pairs - 1) / pairs;
    const int64_t split_rounds = (split_tiles * s + pairs - 1) / pairs;
    return whole_rounds * (num_kb + 16) + split_rounds * ((num_kb + s - 1) / s + 16);
  };
  GemmSplit best{1, 0};
  int64_t best_cost = cost(tiles, 0, 1);
  const int64_t leftover = tiles % pairs;
  for (int s = 2; s <= kGemmMaxTailSplit && num_kb / s >= 8; ++s) {
    if (s <= kGemmMaxSplit) {
      const int64_t c = cost(0, tiles, s);
      if (c < best_cost) {
        best_cost = c;
        best = GemmSplit{s, static_cast<int>(tiles)};
      }
    }
    if (leftover > 0 && leftover < tiles && num_kb / s >= 24) {
      const int64_t c = cost(tiles - leftover, leftover, s);
      if (c < best_cost) {
        best_cost = c;
        best = GemmSplit{s, static_cast<int>(leftover)};
      }
    }
  }
  return best;
}

cudaError_t launch_gemm_decomp(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& a, int num_sms,
                               bool pdl, cudaStream_t stream) {
  const bool bias = a.bias != nullptr;
  if (a.split > 1)
    return bias ? launch_t<true, true>(tmA, tmB, a, num_sms, pdl, stream)
                : launch_t<false, true>(tmA, tmB, a, num_sms, pdl, stream);
  return bias ? launch_t<true, false>(tmA, tmB, a, num_sms, pdl, stream)
              : launch_t<false, false>(tmA, tmB, a, num_sms, pdl, stream);
}

}  // namespace i8mm
