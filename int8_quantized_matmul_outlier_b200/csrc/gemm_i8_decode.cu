// Decode-shape variant of the fused int8 GEMM (few tokens, M <= 64) for sm_100a.
//
//   Y[m,n] = fp16( Acc[m,n] / (c_x[m] c_w[n]) + sum_{k in O} X[m,k] W[k,n] [+ b[n]] ),  Acc = Xq Wq^T
//
// Method: as the prefill kernel ("LLM.int8() — 大模型激活值里藏着几个超大异常通道",
// 方法1 and 方法2; the Fig. 2 caption of the AI 十大核心论文解读 article).
//
// With a handful of tokens the contraction is bound by streaming the int8
// weight from HBM, so the operands are swapped: a 128-row tile of Wq (128
// output columns n) takes the MMA's M slot and the MP padded tokens its N slot,
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
// Warps: 0 TMA producer (weight tile + token tile per stage, 6-deep ring,
// weight loads marked evict-first in L2; the first weight tiles are issued
// before waiting on the activation pass), 1 MMA issuer and TMEM owner (double-buffered 128 x MP int32
// accumulator), 2-9 epilogue (one output column n per thread, half of the
// tokens: two warps share each TMEM lane quarter).
// Every wait is bounded; a timeout sets the status word and the CTA exits.
#include "kernels.cuh"
#include "ptx.cuh"

#include <algorithm>

namespace i8mm {
namespace {

constexpr int DBM = 128;  // weight rows (output columns) per tile: the MMA M
constexpr int DBK = 128;  // K bytes per stage
// Six stages of weight tiles in flight per SM measured faster than deeper
// rings (4: slower, 11: 12% slower): more outstanding reads only congest HBM.
constexpr int D_STAGES = 6;
constexpr int D_OUT_STAGE = 128;  // outliers whose activations (and indices) are staged in smem
constexpr int D_EPI = 256;  // epilogue threads: eight warps
constexpr int D_THREADS = 64 + D_EPI;

template <int MP>
struct DCfg {
  static constexpr int W_BYTES = DBM * DBK;
  static constexpr int X_BYTES = MP * DBK;
  static constexpr int STAGE = W_BYTES + X_BYTES;
  static constexpr int STAGES = D_STAGES;
  static constexpr int BAR_OFF = STAGES * STAGE;
  static constexpr int NBARS = 2 * STAGES + 5;
  static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
  static constexpr int XO_OFF = (MISC_OFF + 32 + 15) & ~15;        // half [D_OUT_STAGE][64]
  static constexpr int RX_OFF = XO_OFF + D_OUT_STAGE * 64 * 2;     // float [64]
  static constexpr int IDX_OFF = RX_OFF + 64 * 4;                  // int [D_OUT_STAGE]
  static constexpr int SMEM = IDX_OFF + D_OUT_STAGE * 4 + 1024;
  // outlier weight values prefetched into registers per segment
  static constexpr int WCAP = 16;
  static constexpr int TMEM_COLS = 2 * MP < 32 ? 32 : 2 * MP;
  static constexpr uint32_t IDESC = idesc_i8(DBM, MP);
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

template <int MP>
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
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);
  volatile int* s_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 8);
  __half* xo_s = reinterpret_cast<__half*>(smem + C::XO_OFF);
  float* rx_s = reinterpret_cast<float*>(smem + C::RX_OFF);
  int* idx_s = reinterpret_cast<int*>(smem + C::IDX_OFF);

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
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
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
      dpdl_wait();
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
    const int q = warp & 3;
    const int m0 = ((warp - 2) >> 2) * HM;
    const int n_local = q * 32 + lane;
    const int et = threadIdx.x - 64;  // 0 .. D_EPI-1
    dpdl_wait();  // count, idx, X_OT and c_x come from the activation pass
    const int cnt = *a.count;
    const int cs = min(cnt, D_OUT_STAGE);
    for (int e = et; e < cs * M; e += D_EPI) {
      const int o = e / M, m = e % M;
      xo_s[o * 64 + m] = a.X_OT[static_cast<size_t>(o) * a.ld_xo + m];
    }
    for (int o = et; o < cs; o += D_EPI) idx_s[o] = a.idx[o];
    if (et < M) {
      const float c = a.c_x[et];
      rx_s[et] = c == 0.0f ? 0.0f : __frcp_rn(c);
    }
    dbar_sync(1, D_EPI);
    int lt = 0;
    for (long long u = u_begin; u < u_end; ++lt) {
      const Seg sg = segment_at(u, u_end, num_kb);
      u += sg.kb1 - sg.kb0;
      const int buf = lt & 1;
      const uint32_t use = static_cast<uint32_t>(lt >> 1);
      const int n = sg.nb * DBM + n_local;
      const bool n_ok = n < N;
      // outlier weight values of this column: they do not depend on the
      // accumulator, so load them while the tensor cores still work
      float wo[C::WCAP];
#pragma unroll
      for (int o = 0; o < C::WCAP; ++o)
        wo[o] = (o < cs && n_ok) ? __half2float(a.W[static_cast<size_t>(idx_s[o]) * N + n]) : 0.0f;
      // all lanes wait; the decision to go on is then made once for all warps
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&tfull[buf], use & 1u, tmo, abort_flag));
      if (!ok && lane == 0) dfail(a, abort_flag);
      dbar_sync(1, D_EPI);
      if (et == 0) *s_flag = *abort_flag ? 0 : 1;
      dbar_sync(1, D_EPI);
      if (!*s_flag) continue;
      tc_fence_after();
      uint32_t r[HM];
      const uint32_t t =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(buf * MP + m0);
      if constexpr (HM >= 16) {
#pragma unroll
        for (int j = 0; j < HM / 16; ++j) tmem_ld_32x32b_x16(t + 16 * j, r + 16 * j);
      } else {
        tmem_ld_32x32b_x8(t, r);
      }
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[buf]);

      if (sg.kb0 != 0) {
        // a later piece of a split n block: add into the global sums and
        // count the k steps for the block's owner
        if (n_ok) {
#pragma unroll
          for (int j = 0; j < HM; ++j)
            if (m0 + j < M) atomicAdd(a.part + static_cast<size_t>(m0 + j) * N + n, static_cast<int>(r[j]));
        }
        __threadfence();
        dbar_sync(1, D_EPI);
        if (et == 0 && !a.skip_arrival) atomicAdd(a.ticket + sg.nb, static_cast<unsigned>(sg.kb1 - sg.kb0));
        continue;
      }
      if (sg.kb1 != num_kb) {
        // the owner of a split n block: wait for the other pieces' k steps,
        // then add their sums
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
        if (!got) continue;
        if (n_ok) {
          // all loads first: a store between them would serialise the round
          // trips (the compiler cannot tell the addresses apart)
          int32_t v[HM];
#pragma unroll
          for (int j = 0; j < HM; ++j)
            v[j] = m0 + j < M ? __ldcg(a.part + static_cast<size_t>(m0 + j) * N + n) : 0;
#pragma unroll
          for (int j = 0; j < HM; ++j)
            if (m0 + j < M) a.part[static_cast<size_t>(m0 + j) * N + n] = 0;
#pragma unroll
          for (int j = 0; j < HM; ++j) r[j] = static_cast<uint32_t>(static_cast<int>(r[j]) + v[j]);
        }
        if (et == 0) a.ticket[sg.nb] = 0u;
      }
      if (!n_ok) continue;
      // dequantise, add the fp16 outlier product, write fp16 (coalesced over n)
      const float rw = __ldg(a.inv_cw + n);
      const float bn = a.bias != nullptr ? __half2float(a.bias[n]) : 0.0f;
      float y[HM];
#pragma unroll
      for (int j = 0; j < HM; ++j)
        y[j] = m0 + j < M
                   ? __fadd_rn(__fmul_rn(__fmul_rn(__int2float_rn(static_cast<int>(r[j])), rx_s[m0 + j]), rw), bn)
                   : 0.0f;
#pragma unroll
      for (int o = 0; o < C::WCAP; ++o)
        if (o < cs) {
#pragma unroll
          for (int j = 0; j < HM; ++j)
            if (m0 + j < M) y[j] = __fmaf_rn(__half2float(xo_s[o * 64 + m0 + j]), wo[o], y[j]);
        }
      // outliers past WCAP: their weight values in batches (eight, four
      // with 64 tokens, where registers are scarcer), the loads of a batch
      // all in flight before its FMAs (still in ascending o)
      constexpr int OB = MP >= 64 ? 4 : 8;
      for (int o0 = C::WCAP; o0 < cnt; o0 += OB) {
        float w8[OB];
#pragma unroll
        for (int u = 0; u < OB; ++u) {
          const int o = o0 + u;
          w8[u] = o < cnt ? __half2float(a.W[static_cast<size_t>(o < cs ? idx_s[o] : __ldg(a.idx + o)) * N + n])
                          : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < OB; ++u) {
          const int o = o0 + u;
          if (o < cnt) {
#pragma unroll
            for (int j = 0; j < HM; ++j)
              if (m0 + j < M) {
                const float xo = o < cs ? __half2float(xo_s[o * 64 + m0 + j])
                                        : __half2float(a.X_OT[static_cast<size_t>(o) * a.ld_xo + m0 + j]);
                y[j] = __fmaf_rn(xo, w8[u], y[j]);
              }
          }
        }
      }
#pragma unroll
      for (int j = 0; j < HM; ++j)
        if (m0 + j < M) a.Y[static_cast<size_t>(m0 + j) * N + n] = __float2half_rn(y[j]);
      if (a.acc_dump != nullptr) {
#pragma unroll
        for (int j = 0; j < HM; ++j)
          if (m0 + j < M) a.acc_dump[static_cast<size_t>(m0 + j) * N + n] = static_cast<int32_t>(r[j]);
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

template <int MP>
cudaError_t launch_decode_t(const CUtensorMap& tmW, const CUtensorMap& tmX, const DecodeArgs& a, int num_sms,
                            bool pdl, cudaStream_t stream) {
  using C = DCfg<MP>;
  static unsigned long long attr_set = 0;  // one bit per device
  int dev = 0;
  cudaGetDevice(&dev);
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_set & bit)) {
    cudaError_t e = cudaFuncSetAttribute(gemm_i8_decode_kernel<MP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::SMEM);
    if (e != cudaSuccess) return e;
    attr_set |= bit;
  }
  const long long total = static_cast<long long>((a.N + DBM - 1) / DBM) * ((a.K + DBK - 1) / DBK);
  const int grid = static_cast<int>(std::max(1LL, std::min<long long>(total, num_sms)));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(D_THREADS);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, gemm_i8_decode_kernel<MP>, tmW, tmX, a);
}

}  // namespace

int decode_padded_tokens(int64_t M) { return M <= 16 ? 16 : (M <= 32 ? 32 : 64); }

cudaError_t launch_gemm_decode(const CUtensorMap& tmW, const CUtensorMap& tmX, const DecodeArgs& a, int num_sms,
                               bool pdl, cudaStream_t stream) {
  switch (decode_padded_tokens(a.M)) {
    case 16: return launch_decode_t<16>(tmW, tmX, a, num_sms, pdl, stream);
    case 32: return launch_decode_t<32>(tmW, tmX, a, num_sms, pdl, stream);
    default: return launch_decode_t<64>(tmW, tmX, a, num_sms, pdl, stream);
  }
}

}  // namespace i8mm
