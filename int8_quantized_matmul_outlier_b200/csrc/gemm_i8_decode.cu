// Decode-shape variant of the fused int8 GEMM (few tokens, M <= 128) for sm_100a.
//
//   Y[m,n] = fp16( Acc[m,n] / (c_x[m] c_w[n]) + sum_{k in O} X[m,k] W[k,n] [+ b[n]] ),  Acc = Xq Wq^T
//
// Method: as the prefill kernel ("LLM.int8() — 大模型激活值里藏着几个超大异常通道",
// 方法1 and 方法2; the Fig. 2 caption of the AI 十大核心论文解读 article).
//
// With a handful of tokens the contraction is bound by streaming the int8
// weight from HBM, so the operands are swapped: a 128-row tile of Wq (128
// output columns n) takes the MMA's M slot and the MP padded tokens (16, 32,
// 64 or 128) its N slot,
// D^T[n, m] = sum_k Wq[n, k] Xq[m, k]  (tcgen05.mma kind::i8, 128 x MP x 32).
//
// Work split (stream-K): the N/128 x K/128 sequence of (n block, k block)
// steps is cut into gridDim.x equal contiguous ranges, one per persistent CTA,
// so every SM streams the same number of weight bytes.  A range covers whole
// n blocks (finished straight from TMEM) and at most two partial ones.  The
// piece of a split n block that holds k block 0 owns it: it is the last
// segment of its CTA's range, while the other pieces are first segments of
// the following CTAs, done early.  Those add their int32 sums exactly into a
// global buffer and count their k steps on the block's ticket; the owner
// waits (bounded) until the ticket shows the rest of K, adds the buffer to
// its own sums, clears buffer and ticket, and finishes the block.  Owners
// wait only on pieces that wait on nothing.  Integer sums make the result
// independent of order.
//
// Activation pass in the same launch (for K up to 16384): the CTAs are
// co-resident (a cooperative launch), and CTA c of G takes the columns
// [8 v0, 8 v1) of X, v0 = c nvec / G (nvec = K/8).  Its epilogue warps, idle
// until the first accumulator is ready, load X[0..M, slice] once and
//   1. flag the slice's outlier columns, exactly: all M rows are at hand;
//   2. take each row's absmax over the slice's columns outside O, fold it
//      into a global per-row maximum (atomicMax on the magnitude bits) and
//      OR the flags into a global bitmask;
//   3. meet the other CTAs at a grid barrier; then c_x = 127/absmax of every
//      row, the codes of the slice (outlier columns 0), and, from the
//      bitmask's bits before the slice, the positions in O of the slice's
//      outlier columns: idx and X_OT for them;
//   4. meet at a second grid barrier, after which the producer loads the
//      token tiles of Xq with TMA.
// Meanwhile the producer has issued the first ring of weight tiles.
// Prefetching the next ones into L2 as well (24 tiles per CTA) measured
// slower: it delayed the first grid barrier by about 2 us (the release of
// the arrival waits for the CTA's outstanding memory operations).  The barrier state (bitmasks, arrival counters and the
// generation word) is the one the separate activation pass keeps, with the
// same rule: the launch of generation g uses the parity-g buffers, finds
// them zero, and clears the parity-(g+1) ones for the next launch.
//
// Outlier product on the tensor cores: for every segment that writes Y, the
// epilogue warps stage W[O, n block] and X[:, O] as fp16 K-major operands, a
// chunk of kOutMma outliers at a time (transposed in registers from
// coalesced 16-byte loads), while the int8 part runs; after it, the MMA warp
// adds D_O^T[n, m] = sum_{o} W[O_o, n] X[m, O_o] into a third, fp32 TMEM
// accumulator (kind::f16, 128 x MP x 16 per instruction), which the
// epilogue adds to the dequantised int8 part.
//
// Warps: 0 TMA producer (weight tile + token tile per stage, 6-deep ring,
// weight loads marked evict-first in L2; the first ring of weight tiles is
// loaded before waiting on the activation pass), 1 MMA issuer and TMEM owner (double-buffered 128 x MP int32
// accumulator, 128 x MP fp32 outlier product), 2-9 epilogue (one output
// column n per thread, half of the tokens: two warps share each TMEM lane
// quarter) and outlier staging.
// Every wait is bounded; a timeout sets the status word and the CTA exits.
#include "actq.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

#include <algorithm>

namespace i8mm {
namespace {

constexpr int DBM = 128;  // weight rows (output columns) per tile: the MMA M
constexpr int DBK = 128;  // K bytes per stage
// Six stages of weight tiles in flight per SM measured faster than deeper
// rings (4: slower, 11: 12% slower): more outstanding reads only congest HBM.
// With 128 tokens a stage holds 32 KB, and five fit.
constexpr int D_STAGES = 6;
constexpr int D_STAGES_128 = 5;
constexpr int D_OUT_STAGE = 128;  // outliers whose indices are staged in smem
constexpr int D_EPI = 256;  // epilogue threads: eight warps
constexpr int D_THREADS = 64 + D_EPI;

template <int MP>
struct DCfg {
  static constexpr int W_BYTES = DBM * DBK;
  static constexpr int X_BYTES = MP * DBK;
  static constexpr int STAGE = W_BYTES + X_BYTES;
  static constexpr int STAGES = MP > 64 ? D_STAGES_128 : D_STAGES;
  // operands of the outlier product, one chunk of kOutMma outliers, fp16,
  // K-major rows of 128 bytes with the 128-byte swizzle: A = W[O, n block]
  // (128 columns n), B = X[:, O] (MP tokens)
  static constexpr int OA_OFF = STAGES * STAGE;
  static constexpr int OB_OFF = OA_OFF + DBM * 128;
  static constexpr int BAR_OFF = OB_OFF + MP * 128;
  static constexpr int NBARS = 2 * STAGES + 8;
  static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
  // The fused activation pass's slice of X, uint4 [MP rows][16 vectors],
  // lives in the outlier operand blocks (16 KB + MP 128 bytes >= MP 256
  // bytes): it is dead before the first outlier chunk is staged.
  static constexpr int XS_OFF = OA_OFF;
  static_assert(DBM * 128 + MP * 128 >= MP * 16 * 16, "the X slice fits the outlier operand blocks");
  static constexpr int RX_OFF = (MISC_OFF + 32 + 15) & ~15;        // float [MP]
  static constexpr int IDX_OFF = RX_OFF + MP * 4;                  // int [D_OUT_STAGE]
  static constexpr int CX_OFF = IDX_OFF + D_OUT_STAGE * 4;         // float [MP]: c_x (fused)
  static constexpr int FL_OFF = CX_OFF + MP * 4;                   // u32 [16]: flags per vector (fused)
  static constexpr int OL_OFF = FL_OFF + 16 * 4;                   // u32 [128]: the slice's outliers (fused)
  static constexpr int RED_OFF = OL_OFF + 128 * 4;                 // u32 [16]: reductions (fused)
  static constexpr int SMEM = RED_OFF + 16 * 4 + 1024;
  // TMEM: two int32 accumulators (double buffer) and the fp32 outlier
  // product, MP columns each, in a power-of-two allocation
  static constexpr int TMEM_COLS =
      3 * MP <= 32 ? 32 : (3 * MP <= 64 ? 64 : (3 * MP <= 128 ? 128 : (3 * MP <= 256 ? 256 : 512)));
  static constexpr uint32_t IDESC = idesc_i8(DBM, MP);
  static constexpr uint32_t IDESC_F16 = idesc_f16_f32(DBM, MP);
  static_assert(OA_OFF % 1024 == 0 && OB_OFF % 1024 == 0, "outlier operands 1024-byte aligned");
  static_assert(STAGE % 1024 == 0, "stages stay 1024-byte aligned for the 128B swizzle");
  static_assert(SMEM <= 232448, "fits the 227 KB of shared memory per block");
};

__device__ __forceinline__ void dpdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void dbar_sync(uint32_t id, uint32_t n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ void dfail(const DecodeArgs& a, volatile int* abort_flag) {
  *abort_flag = 1;
  atomicOr(a.status, kStatusTimeout);
}

// Persistent CTAs of the decode GEMM: one per SM, at most one per
// (n block, k block) step.
int64_t decode_grid(int64_t N, int64_t K, int num_sms) {
  const int64_t total = ((N + DBM - 1) / DBM) * ((K + DBK - 1) / DBK);
  return std::max<int64_t>(1, std::min<int64_t>(total, num_sms));
}

// Grid barrier of the fused activation pass (one thread per CTA): optionally
// counts this CTA with a release add, then waits (acquire) until the counter
// reaches `target`; false once timeout_ns have passed.
__device__ __forceinline__ bool grid_wait(uint32_t* ctr, uint32_t target, bool arrive, uint64_t timeout_ns) {
  if (arrive) red_release_add_gpu(ctr, 1u);
  if (ld_acquire_gpu_u32(ctr) >= target) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (ld_acquire_gpu_u32(ctr) >= target) return true;
    if ((it & 15u) == 0 && global_timer_ns() - t0 > timeout_ns) return false;
  }
}

// One segment of a CTA's range: n block `nb`, k blocks [kb0, kb1).
struct Seg {
  int nb, kb0, kb1;
};

__device__ __forceinline__ Seg segment_at(long long u, long long u_end, int num_kb) {
  Seg s;
  s.nb = static_cast<int>(u / num_kb);
  s.kb0 = static_cast<int>(u % num_kb);
  const long long seg_end = min(u_end, static_cast<long long>(s.nb + 1) * num_kb);
  s.kb1 = s.kb0 + static_cast<int>(seg_end - u);
  return s;
}

template <int MP, bool FUSED>
__global__ void __launch_bounds__(D_THREADS, 1)
    gemm_i8_decode_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                          const DecodeArgs a) {
  using C = DCfg<MP>;
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* act_ready = drain + 1;  // fused: the token tiles of Xq may be loaded
  uint64_t* ofull = act_ready + 1;   // an outlier chunk is staged (one arrival per epilogue warp)
  uint64_t* oempty = ofull + 1;      // the tensor cores are done with the staged chunk
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);
  volatile int* s_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 8);
  float* rx_s = reinterpret_cast<float*>(smem + C::RX_OFF);
  int* idx_s = reinterpret_cast<int*>(smem + C::IDX_OFF);
  float* cx_s = reinterpret_cast<float*>(smem + C::CX_OFF);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int M = a.M, N = a.N, K = a.K;
  const int n_blks = (N + DBM - 1) / DBM;
  const int num_kb = (K + DBK - 1) / DBK;
  const long long total = static_cast<long long>(n_blks) * num_kb;
  const long long u_begin = total * blockIdx.x / gridDim.x;
  const long long u_end = total * (blockIdx.x + 1) / gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], D_EPI / 32);
    }
    mbar_init(drain, 1);
    mbar_init(act_ready, 1);
    mbar_init(ofull, D_EPI / 32);
    mbar_init(oempty, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  // fused: the epilogue warps start loading their slice of X right away
  // (vectors e = et + j D_EPI of the [M][16] slice; see the activation pass)
  constexpr int XR = MP * 16 / D_EPI > 0 ? MP * 16 / D_EPI : 1;
  uint4 xr[XR];
  int xv0 = 0, xnv = 0;
  if constexpr (FUSED) {
    const int nvec = K >> 3;
    xv0 = static_cast<int>(static_cast<long long>(nvec) * blockIdx.x / gridDim.x);
    xnv = static_cast<int>(static_cast<long long>(nvec) * (blockIdx.x + 1) / gridDim.x) - xv0;  // <= 16
    if (warp >= 2) {
      const uint4* X4 = reinterpret_cast<const uint4*>(a.X);
#pragma unroll
      for (int j = 0; j < XR; ++j) {
        const int e = static_cast<int>(threadIdx.x) - 64 + j * D_EPI, m = e >> 4, v = e & 15;
        xr[j] = (m < M && v < xnv) ? __ldg(X4 + static_cast<size_t>(m) * nvec + xv0 + v) : make_uint4(0, 0, 0, 0);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const unsigned long long tmo = a.timeout_ns;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ TMA producer
      uint32_t issued_mask = 0, issued_phase = 0;
      bool ok = true;
      // the weight is read exactly once: do not let it push other data out of L2
      const uint64_t wpol = l2_policy_evict_first();
      // weight tiles do not depend on the activation pass: issue the first
      // ring's worth before waiting for it (every stage starts empty)
      const int pre = static_cast<int>(min(static_cast<long long>(STAGES), u_end - u_begin));
      for (int i = 0; i < pre; ++i) {
        const long long uu = u_begin + i;
        const int nb = static_cast<int>(uu / num_kb), kb = static_cast<int>(uu % num_kb);
        mbar_arrive_expect_tx(&full[i], C::STAGE);
        tma_load_2d_hint(smem + i * C::STAGE, &tmW, &full[i], 0, kb * a.N_pad + nb * DBM, wpol);
      }
      if constexpr (FUSED) {
        // Xq is written by the CTAs' activation pass; the epilogue warps
        // signal after its second grid barrier (also when a barrier ran
        // out, with the abort flag set: the token tiles are loaded all the
        // same, so that every issued stage completes)
        if (!mbar_wait(act_ready, 0, 3 * tmo, nullptr)) dfail(a, abort_flag);
        fence_proxy_async_global();
      } else {
        dpdl_wait();
      }
      for (int i = 0; i < pre; ++i) {
        const int kb = static_cast<int>((u_begin + i) % num_kb);
        tma_load_2d(smem + i * C::STAGE + C::W_BYTES, &tmX, &full[i], kb * DBK, 0);
        issued_mask |= 1u << i;
      }
      int stage = pre % STAGES;
      uint32_t phase = pre == STAGES ? 1u : 0u;
      for (long long uu = u_begin + pre; uu < u_end && ok; ++uu) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, tmo, abort_flag)) {
          ok = false;
          break;
        }
        const int nb = static_cast<int>(uu / num_kb), kb = static_cast<int>(uu % num_kb);
        uint8_t* st = smem + stage * C::STAGE;
        mbar_arrive_expect_tx(&full[stage], C::STAGE);
        tma_load_2d_hint(st, &tmW, &full[stage], 0, kb * a.N_pad + nb * DBM, wpol);
        tma_load_2d(st + C::W_BYTES, &tmX, &full[stage], kb * DBK, 0);
        issued_mask |= 1u << stage;
        issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) {
        dfail(a, abort_flag);
        for (int s = 0; s < STAGES; ++s)
          if (issued_mask & (1u << s)) mbar_wait(&full[s], (issued_phase >> s) & 1u, tmo, nullptr);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // -------------------------------------------------------- MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int lt = 0;
      int cnt = -1;             // |O|, read at the first segment that writes Y
      uint32_t orounds = 0;     // outlier chunks issued so far
      const uint32_t d2_tmem = tmem_base + static_cast<uint32_t>(2 * MP);
      for (long long u = u_begin; u < u_end && ok; ++lt) {
        const Seg sg = segment_at(u, u_end, num_kb);
        u += sg.kb1 - sg.kb0;
        const int buf = lt & 1;
        const uint32_t use = static_cast<uint32_t>(lt >> 1);
        if (!mbar_wait(&tempty[buf], (use & 1u) ^ 1u, tmo, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * MP);
        for (int kb = sg.kb0; kb < sg.kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, tmo, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * C::STAGE);
          const uint64_t adesc = smem_desc_k_sw128(sa);
          const uint64_t bdesc = smem_desc_k_sw128(sa + C::W_BYTES);
#pragma unroll
          for (int kk = 0; kk < DBK / 32; ++kk)
            mma_i8(d_tmem, adesc + static_cast<uint64_t>(kk * 2), bdesc + static_cast<uint64_t>(kk * 2), C::IDESC,
                   (kb > sg.kb0 || kk > 0) ? 1u : 0u);
          mma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok && sg.kb0 == 0) {
          // this segment writes Y: the fp16 outlier product into its own
          // accumulator, one staged chunk of kOutMma outliers at a time
          if (cnt < 0) {
            if constexpr (FUSED) {
              if (!mbar_wait(act_ready, 0, 3 * tmo, abort_flag)) ok = false;
            } else {
              dpdl_wait();
            }
            cnt = ok ? __ldcg(a.count) : 0;
          }
          const uint64_t oad = smem_desc_k_sw128(smem_u32(smem + C::OA_OFF));
          const uint64_t obd = smem_desc_k_sw128(smem_u32(smem + C::OB_OFF));
          for (int o0 = 0; o0 < cnt && ok; o0 += kOutMma) {
            if (!mbar_wait(ofull, orounds & 1u, tmo, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const int ks = (min(cnt - o0, kOutMma) + 15) / 16;
            for (int kk = 0; kk < ks; ++kk)
              mma_f16(d2_tmem, oad + static_cast<uint64_t>(kk * 2), obd + static_cast<uint64_t>(kk * 2),
                      C::IDESC_F16, (o0 > 0 || kk > 0) ? 1u : 0u);
            mma_commit(oempty);
            ++orounds;
          }
        }
        if (ok) mma_commit(&tfull[buf]);
      }
      if (!ok) {
        dfail(a, abort_flag);
        mma_commit(drain);
        mbar_wait(drain, 0, tmo, nullptr);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Two warps per TMEM lane quarter (warp w may read lanes 32 (w % 4) ..):
    // warps 2-5 take tokens [0, HM), warps 6-9 tokens [HM, MP).
    constexpr int HM = MP / 2;
    constexpr int HC = HM > 16 ? 16 : HM;  // tokens per chunk of the epilogue
    const int q = warp & 3;
    const int m0 = ((warp - 2) >> 2) * HM;
    const int n_local = q * 32 + lane;
    const int et = threadIdx.x - 64;  // 0 .. D_EPI-1
    if constexpr (FUSED) {
      // ------------------------------------------ activation pass of the slice
      uint4* xs = reinterpret_cast<uint4*>(smem + C::XS_OFF);  // [MP][16] (in the outlier operand blocks)
      uint32_t* fl_s = reinterpret_cast<uint32_t*>(smem + C::FL_OFF);
      uint32_t* ol_s = reinterpret_cast<uint32_t*>(smem + C::OL_OFF);
      uint32_t* red_s = reinterpret_cast<uint32_t*>(smem + C::RED_OFF);
      volatile uint32_t* s_gen = reinterpret_cast<volatile uint32_t*>(smem + C::MISC_OFF + 12);
      volatile int* s_nloc = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 16);
      const int G = static_cast<int>(gridDim.x), cta = static_cast<int>(blockIdx.x);
      const int KW = (K + 31) >> 5;
      const int v0 = xv0, nv = xnv;
      if (et == 0) *s_gen = *reinterpret_cast<volatile uint32_t*>(a.sync + 2);
      // (0) X[0..M, 8 v0 .. 8 (v0 + nv)): 16 vectors of 8 columns per row,
      //     loaded before the setup barrier
#pragma unroll
      for (int j = 0; j < XR; ++j) {
        const int e = et + j * D_EPI;
        if (e < M * 16) xs[e] = xr[j];
      }
      dbar_sync(1, D_EPI);
      // (1) outlier flags of the slice's columns (one thread per column, one
      //     flag byte per vector)
      {
        bool out = false;
        if (et < nv * 8) {
          const unsigned short* hs = reinterpret_cast<const unsigned short*>(xs) + et;
          uint32_t mx = 0u;
          for (int m = 0; m < M; ++m) mx = max(mx, static_cast<uint32_t>(hs[m * 128] & 0x7fffu));
          out = a.thr < 0 || mx > static_cast<uint32_t>(a.thr);
        }
        if (et < 128) {  // whole warps: columns et of vectors et / 8
          const uint32_t b = __ballot_sync(0xffffffffu, out);
          if (lane < 4) fl_s[(et >> 5) * 4 + lane] = (b >> (8 * lane)) & 0xffu;
        }
      }
      dbar_sync(1, D_EPI);
      // (2) the flags into this generation's bitmask; per row, the absmax over
      //     the slice's columns outside O into the global maximum (16 lanes
      //     per row, reduced by shuffles)
      const uint32_t gen = *s_gen;
      uint32_t* gmask = a.omask + static_cast<size_t>(gen & 1u) * KW;
      if (et < nv && fl_s[et] != 0u) atomicOr(gmask + ((v0 + et) >> 2), fl_s[et] << (((v0 + et) & 3) * 8));
      for (int base = 0; base < M * 16; base += D_EPI) {
        const int e = base + et, m = e >> 4, v = e & 15;
        uint32_t r = 0u;
        if (e < M * 16 && v < nv) r = max_pair(masked_absmax2(0u, xs[e], fl_s[v]));
        r = max(r, __shfl_xor_sync(0xffffffffu, r, 8));
        r = max(r, __shfl_xor_sync(0xffffffffu, r, 4));
        r = max(r, __shfl_xor_sync(0xffffffffu, r, 2));
        r = max(r, __shfl_xor_sync(0xffffffffu, r, 1));
        if (e < M * 16 && v == 0 && r != 0u) atomicMax(a.rowmax + m * kRowMaxStride, r);
      }
      // (3) grid barrier: every CTA's flags and row maxima are in
      dbar_sync(1, D_EPI);
      if (et == 0) {
        const bool arrive = !(a.skip_barrier && cta == 0);
        const bool ok1 = grid_wait(a.sync + (gen & 1u), static_cast<uint32_t>(G), arrive, tmo);
        if (!ok1) dfail(a, abort_flag);
        *s_flag = ok1 ? 1 : 0;
      }
      dbar_sync(1, D_EPI);
      if (*s_flag) {
        // (4) the row maxima and the bitmask, read together: the scales of
        //     all rows (CTA 0 writes them out), and the position in O of the
        //     slice's first column, i.e. the bits of the bitmask before it
        //     (for CTA 0 also |O|: all of them)
        const uint32_t rmax = et < M ? __ldcg(a.rowmax + et * kRowMaxStride) : 0u;
        const int wf = v0 >> 2;
        const uint32_t below = (1u << ((v0 & 3) * 8)) - 1u;
        uint32_t before = 0u, total = 0u;
        for (int w = et; w < KW; w += D_EPI) {
          const uint32_t bits = __ldcg(gmask + w);
          total += __popc(bits);
          before += w < wf ? __popc(bits) : (w == wf ? __popc(bits & below) : 0);
        }
        if (et < M) {
          const float c = scale_from_absmax_bits(rmax);
          cx_s[et] = c;
          if (cta == 0) a.c_x_out[et] = c;
        }
        before = __reduce_add_sync(0xffffffffu, before);
        total = __reduce_add_sync(0xffffffffu, total);
        if (lane == 0) {
          red_s[2 * (warp - 2)] = before;
          red_s[2 * (warp - 2) + 1] = total;
        }
        dbar_sync(1, D_EPI);
        // the codes of the slice, outlier columns 0
        for (int e = et; e < M * 16; e += D_EPI) {
          const int m = e >> 4, v = e & 15;
          if (v < nv) {
            const uint32_t fl = fl_s[v];
            uint2 q = quant8_fma(xs[e], cx_s[m]);
            q.x &= ~expand_nibble(fl & 0xfu);
            q.y &= ~expand_nibble(fl >> 4);
            *reinterpret_cast<uint2*>(a.Xq_out + static_cast<size_t>(m) * K + static_cast<size_t>(v0 + v) * 8) = q;
          }
        }
        // (5) the slice's outlier columns: idx and their local list
        if (et == 0) {
          uint32_t o = 0u, n_all = 0u;
          for (int u = 0; u < D_EPI / 32; ++u) {
            o += red_s[2 * u];
            n_all += red_s[2 * u + 1];
          }
          int n = 0;
          for (int v = 0; v < nv; ++v) {
            uint32_t b = fl_s[v];
            while (b != 0u) {
              const int q = __ffs(static_cast<int>(b)) - 1;
              b &= b - 1u;
              a.idx_out[o] = (v0 + v) * 8 + q;
              ol_s[n++] = (o << 8) | static_cast<uint32_t>(v * 8 + q);
              ++o;
            }
          }
          *s_nloc = n;
          if (cta == 0) *a.count_out = static_cast<int32_t>(n_all);
        }
        dbar_sync(1, D_EPI);
        // (6) X_OT for the slice's outlier columns
        const int n_loc = *s_nloc;
        for (int e = et; e < n_loc * M; e += D_EPI) {
          const int j = e / M, m = e - j * M;
          const uint32_t oc = ol_s[j];
          a.X_OT_out[static_cast<size_t>(oc >> 8) * a.ld_xo + m] =
              reinterpret_cast<const __half*>(xs)[m * 128 + static_cast<int>(oc & 255u)];
        }
        // the next launch's bitmask and arrival counter start at zero
        if (cta == 0) {
          uint32_t* next = a.omask + static_cast<size_t>((gen + 1u) & 1u) * KW;
          for (int w = et; w < KW; w += D_EPI) next[w] = 0u;
          if (et == 0) a.sync[(gen + 1u) & 1u] = 0u;
        }
        fence_proxy_async_global();  // other CTAs read these codes with TMA
        // (7) second grid barrier: Xq, c_x, idx, count and X_OT are out
        dbar_sync(1, D_EPI);
        if (et == 0) {
          const bool ok2 = grid_wait(a.sync + (gen & 1u), 2u * static_cast<uint32_t>(G), true, tmo);
          if (!ok2) dfail(a, abort_flag);
          else if (cta == 0) a.sync[2] = gen + 1u;
          *s_flag = ok2 ? 1 : 0;
        }
        dbar_sync(1, D_EPI);
        // every CTA read the row maxima before it arrived
        if (*s_flag && cta == 0 && et < kDecodeMaxM) a.rowmax[et * kRowMaxStride] = 0u;
      }
      if (et == 0) mbar_arrive(act_ready);
    } else {
      dpdl_wait();  // count, idx, X_OT and c_x come from the activation pass
    }
    const int cnt = __ldcg(a.count);
    const int cs = min(cnt, D_OUT_STAGE);
    for (int o = et; o < cs; o += D_EPI) idx_s[o] = __ldcg(a.idx + o);
    if (et < M) {
      const float c = FUSED ? cx_s[et] : __ldcg(a.c_x + et);
      rx_s[et] = c == 0.0f ? 0.0f : __frcp_rn(c);
    }
    dbar_sync(1, D_EPI);
    // Stages outliers [o0, o0 + kOutMma) of the product's operands for n
    // block nb: A = W[O, n block] (128 rows n), B = X_OT^T (MP rows m).
    // Thread et takes the 8 x 8 block of rows 8 (b >> 3) .. +7 and outliers
    // 8 (b & 7) .. +7 (b = et: A, b = et - 128: B): eight 16-byte loads along
    // the rows, transposed in registers into eight 16-byte pieces of the
    // K-major 128-byte-swizzled layout (piece j of row r at j ^ (r % 8),
    // groups of 8 rows 1024 bytes apart).  Only the 16-outlier steps the
    // product reads are written; zero past |O| and past M or N.
    auto stage_outliers = [&](int o0, int nb) {
      const int no = min(cnt - o0, kOutMma);
      const int n_og = 2 * ((no + 15) / 16);
      const bool isA = et < DBM;
      const int b = isA ? et : et - DBM;
      if (b >= (isA ? DBM : MP)) return;
      const int og = b & 7, rg = b >> 3;
      if (og >= n_og) return;
      const int r0 = isA ? nb * DBM + 8 * rg : 8 * rg;  // first column n (A) or token m (B)
      const int lim = isA ? N : M;
      uint4 v[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int o = o0 + 8 * og + r;
        v[r] = make_uint4(0u, 0u, 0u, 0u);
        if (o < cnt && r0 < lim) {
          if (isA) {
            const int row = o < cs ? idx_s[o] : __ldcg(a.idx + o);
            v[r] = __ldg(reinterpret_cast<const uint4*>(a.W + static_cast<size_t>(row) * N + r0));
          } else {
            v[r] = __ldcg(reinterpret_cast<const uint4*>(a.X_OT + static_cast<size_t>(o) * a.ld_xo + r0));
          }
        }
      }
      if (r0 + 8 > lim) {  // columns past N or tokens past M: zero
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
      uint4 tv[8];
      transpose8x8_b16(v, tv);
      uint8_t* blk = smem + (isA ? C::OA_OFF : C::OB_OFF) + rg * 1024;
#pragma unroll
      for (int i = 0; i < 8; ++i) *reinterpret_cast<uint4*>(blk + i * 128 + ((og ^ i) << 4)) = tv[i];
    };
    uint32_t orounds = 0;  // outlier chunks staged so far
    int lt = 0;
    for (long long u = u_begin; u < u_end; ++lt) {
      const Seg sg = segment_at(u, u_end, num_kb);
      u += sg.kb1 - sg.kb0;
      const int buf = lt & 1;
      const uint32_t use = static_cast<uint32_t>(lt >> 1);
      const int n = sg.nb * DBM + n_local;
      const bool n_ok = n < N;
      const bool writer = sg.kb0 == 0;  // this segment writes Y
      // the outlier product's operands, while the tensor cores work on the
      // int8 part: chunk by chunk, each once the previous one is consumed
      // (the previous segment's product was read from TMEM before this)
      if (writer && cnt > 0) {
        for (int o0 = 0; o0 < cnt; o0 += kOutMma) {
          if (orounds > 0) {
            const bool okw = __all_sync(0xffffffffu, mbar_wait(oempty, (orounds - 1) & 1u, tmo, abort_flag));
            if (!okw) {
              if (lane == 0) dfail(a, abort_flag);
              break;
            }
          }
          stage_outliers(o0, sg.nb);
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(ofull);
          ++orounds;
        }
      }
      // all lanes wait; the decision to go on is then made once for all warps
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&tfull[buf], use & 1u, tmo, abort_flag));
      if (!ok && lane == 0) dfail(a, abort_flag);
      dbar_sync(1, D_EPI);
      if (et == 0) *s_flag = *abort_flag ? 0 : 1;
      dbar_sync(1, D_EPI);
      if (!*s_flag) continue;
      const bool piece = sg.kb0 != 0;                     // a later piece of a split n block
      const bool split_owner = !piece && sg.kb1 != num_kb;  // the owner of a split n block
      if (split_owner) {
        // wait until the other pieces' k steps are on the block's ticket
        if (et == 0) {
          const unsigned need = static_cast<unsigned>(num_kb - sg.kb1);
          int got = 1;
          if (ld_acquire_gpu_u32(a.ticket + sg.nb) != need) {
            const uint64_t t0 = global_timer_ns();
            for (uint32_t it = 1; ld_acquire_gpu_u32(a.ticket + sg.nb) != need; ++it) {
              if ((it & 15u) == 0 && (*abort_flag || global_timer_ns() - t0 > tmo)) {
                got = 0;
                break;
              }
            }
          }
          if (!got) dfail(a, abort_flag);
          *s_flag = got;
        }
        dbar_sync(1, D_EPI);
        const int got = *s_flag;
        dbar_sync(1, D_EPI);  // s_flag is reused by the next segment
        if (!got) {
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[buf]);
          continue;
        }
      }
      tc_fence_after();
      const uint32_t t =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(buf * MP + m0);
      // the outlier product's accumulator (single-buffered, after the two int32 ones)
      const uint32_t t2 = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(2 * MP + m0);
      const float rw = n_ok ? __ldg(a.inv_cw + n) : 0.0f;
      const bool with_o = writer && cnt > 0;  // the segment has an outlier product
      const float bn = (n_ok && a.bias != nullptr) ? __half2float(a.bias[n]) : 0.0f;
      // the thread's HM tokens in chunks of HC (fewer live registers)
#pragma unroll 1
      for (int c = 0; c < HM / HC; ++c) {
        const int mc = m0 + c * HC;  // first token of the chunk
        uint32_t r[HC], d2[HC];
        if constexpr (HC >= 16) {
#pragma unroll
          for (int j = 0; j < HC / 16; ++j) tmem_ld_32x32b_x16(t + c * HC + 16 * j, r + 16 * j);
        } else {
          tmem_ld_32x32b_x8(t + c * HC, r);
        }
        if (with_o) {  // warp-uniform, like every tcgen05.ld
          if constexpr (HC >= 16) {
#pragma unroll
            for (int j = 0; j < HC / 16; ++j) tmem_ld_32x32b_x16(t2 + c * HC + 16 * j, d2 + 16 * j);
          } else {
            tmem_ld_32x32b_x8(t2 + c * HC, d2);
          }
        }
        tmem_wait_ld();
        if (c == HM / HC - 1) {  // the accumulator buffer is free for the MMA warp
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[buf]);
        }
        if (!n_ok) continue;
        if (piece) {
          // add into the global sums
#pragma unroll
          for (int j = 0; j < HC; ++j)
            if (mc + j < M) atomicAdd(a.part + static_cast<size_t>(mc + j) * N + n, static_cast<int>(r[j]));
          continue;
        }
        if (split_owner) {
          // the other pieces' sums; all loads first: a store between them
          // would serialise the round trips (the compiler cannot tell the
          // addresses apart)
          int32_t v[HC];
#pragma unroll
          for (int j = 0; j < HC; ++j)
            v[j] = mc + j < M ? __ldcg(a.part + static_cast<size_t>(mc + j) * N + n) : 0;
#pragma unroll
          for (int j = 0; j < HC; ++j)
            if (mc + j < M) a.part[static_cast<size_t>(mc + j) * N + n] = 0;
#pragma unroll
          for (int j = 0; j < HC; ++j) r[j] = static_cast<uint32_t>(static_cast<int>(r[j]) + v[j]);
        }
        // dequantise, add the layer bias and the fp16 outlier product (fp32
        // from TMEM), write fp16 (coalesced over n)
        float y[HC];
#pragma unroll
        for (int j = 0; j < HC; ++j)
          y[j] = mc + j < M
                     ? __fadd_rn(__fmul_rn(__fmul_rn(__int2float_rn(static_cast<int>(r[j])), rx_s[mc + j]), rw), bn)
                     : 0.0f;
        if (with_o) {
#pragma unroll
          for (int j = 0; j < HC; ++j) y[j] = __fadd_rn(y[j], __uint_as_float(d2[j]));
        }
#pragma unroll
        for (int j = 0; j < HC; ++j)
          if (mc + j < M) a.Y[static_cast<size_t>(mc + j) * N + n] = __float2half_rn(y[j]);
        if (a.acc_dump != nullptr) {
#pragma unroll
          for (int j = 0; j < HC; ++j)
            if (mc + j < M) a.acc_dump[static_cast<size_t>(mc + j) * N + n] = static_cast<int32_t>(r[j]);
        }
      }
      if (piece) {
        // count the k steps for the block's owner
        __threadfence();
        dbar_sync(1, D_EPI);
        if (et == 0 && !a.skip_arrival) atomicAdd(a.ticket + sg.nb, static_cast<unsigned>(sg.kb1 - sg.kb0));
      } else if (split_owner && et == 0) {
        a.ticket[sg.nb] = 0u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

template <int MP, bool FUSED>
cudaError_t launch_decode_t(const CUtensorMap& tmW, const CUtensorMap& tmX, const DecodeArgs& a, int num_sms,
                            bool pdl, cudaStream_t stream) {
  using C = DCfg<MP>;
  static unsigned long long attr_set = 0;  // one bit per device
  int dev = 0;
  cudaGetDevice(&dev);
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_set & bit)) {
    cudaError_t e = cudaFuncSetAttribute(gemm_i8_decode_kernel<MP, FUSED>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr_set |= bit;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(decode_grid(a.N, a.K, num_sms)));
  cfg.blockDim = dim3(D_THREADS);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attr;
  if (FUSED) {
    attr.id = cudaLaunchAttributeCooperative;  // all CTAs resident at once (grid barriers)
    attr.val.cooperative = 1;
  } else {
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
  }
  cfg.attrs = &attr;
  cfg.numAttrs = (FUSED || pdl) ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, gemm_i8_decode_kernel<MP, FUSED>, tmW, tmX, a);
}

template <bool FUSED>
cudaError_t launch_decode_f(const CUtensorMap& tmW, const CUtensorMap& tmX, const DecodeArgs& a, int num_sms,
                            bool pdl, cudaStream_t stream) {
  switch (decode_padded_tokens(a.M)) {
    case 16: return launch_decode_t<16, FUSED>(tmW, tmX, a, num_sms, pdl, stream);
    case 32: return launch_decode_t<32, FUSED>(tmW, tmX, a, num_sms, pdl, stream);
    case 64: return launch_decode_t<64, FUSED>(tmW, tmX, a, num_sms, pdl, stream);
    default: return launch_decode_t<128, FUSED>(tmW, tmX, a, num_sms, pdl, stream);
  }
}

}  // namespace

int decode_padded_tokens(int64_t M) { return M <= 16 ? 16 : (M <= 32 ? 32 : (M <= 64 ? 64 : 128)); }

bool decode_fused_fits(int64_t M, int64_t K, int64_t N, int num_sms) {
  if (M < 1 || M > kDecodeMaxM || K < 16 || K % 16 != 0 || N < 1 || num_sms < 1) return false;
  const int64_t nvec = K / 8;
  const int64_t G = decode_grid(N, K, num_sms);
  return nvec <= 16 * G;  // every CTA's slice has at most ceil(nvec / G) <= 16 vectors
}

cudaError_t launch_gemm_decode(const CUtensorMap& tmW, const CUtensorMap& tmX, const DecodeArgs& a, int num_sms,
                               bool pdl, cudaStream_t stream) {
  if (a.X != nullptr) {
    if (!decode_fused_fits(a.M, a.K, a.N, num_sms)) return cudaErrorInvalidValue;
    return launch_decode_f<true>(tmW, tmX, a, num_sms, false, stream);
  }
  return launch_decode_f<false>(tmW, tmX, a, num_sms, pdl, stream);
}

}  // namespace i8mm
