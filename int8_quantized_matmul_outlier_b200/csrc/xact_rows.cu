// Activation pass for many rows in one launch: outlier-column detection,
// vector-wise row quantisation and the fp16 outlier gather.
//
//   O      = { j : max_i |X[i,j]| > alpha }                        (ascending)
//   c_x[i] = 127 / max_{j not in O} |X[i,j]|,  Xq = rne(X c_x), 0 on O
//   X_OT[o][i] = X[i, O_o]
//
// Method: "LLM.int8() — 大模型激活值里藏着几个超大异常通道", 方法1 and 方法2;
// "LLM.int8()" (brain.gartu.xyz), "Seuil de détection α"; the Fig. 2 caption
// of the AI 十大核心论文解读 article (split, then scale).
//
// X is read from HBM once.  G co-resident blocks (cooperative launch, one per
// SM); block b owns the R consecutive rows [b R, b R + R).  Each of its NW
// warps takes the rows w, w + NW, ... and streams them through a shared-memory
// slot of its own (one bulk copy and one mbarrier per row), so the warps need
// no block-wide synchronisation while X lands.
//
// A row can be quantised before O is known.  A column is in O exactly when
// one of its entries exceeds alpha, so every entry of a column outside O is
// at most alpha.  The block keeps a bitmask of the columns it has seen an
// entry above alpha in (a subset of O).  Per row, once it has landed, the
// group
//   1. flags the columns of the row's entries above alpha;
//   2. takes S_i = max |X[i,j]| over the columns j not flagged so far (all
//      of these entries are at most alpha); S_i is at least the absmax over
//      the columns outside O, and equal to it unless S_i is reached in an
//      outlier column not flagged yet;
//   3. writes c_x[i] = 127 / S_i and the codes of every column with it.
// A block quantises no row before four of its rows are flagged (fewer if it
// has fewer rows or row groups), so in the pages' activations (a few outlier
// columns, large in most rows) the block's bitmask already holds the outlier
// columns when the rows are quantised; rows are quantised as they land.
// Then the block ORs its bitmask into a global one and meets the other
// blocks at a grid barrier (a release add on an arrival counter, acquire
// polling, bounded by %globaltimer).  After it, with the global bitmask:
//   4. for every outlier column j of slot o and every row i of the block:
//      X_OT[o][i] = X[i,j] and the code of (i, j) is set to 0; a row with an
//      outlier-column entry <= alpha equal to S_i is marked;
//   5. a marked row (S_i may come from an outlier column) is quantised
//      again with the exact absmax over the columns outside O.
// Step 5 is rare, and the work after the barrier is a few scattered
// accesses per outlier column and row.
//
// Counters and bitmasks are double-buffered by a generation word that block
// 0 advances after the barrier, so no launch clears anything and the state
// stays on the device (CUDA-graph replay stays valid).
#include "actq.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

#include <algorithm>
#include <cmath>

namespace i8mm {
namespace {

constexpr int kMaxWarps = 32;
constexpr int kMaxGroups = 15;  // named barriers 1..15, one per row group
constexpr int kFirstRows = 4;   // rows flagged before the block quantises any

// Shared memory of a block: one row slot of 2K bytes and one mbarrier per
// row group, the per-warp partial maxima, the bitmask and its word prefix
// (KW words each), S_i and the mark of step 5 of the R rows.
size_t smem_bytes(int64_t groups, int64_t rows, int64_t K) {
  const int64_t KW = (K + 31) / 32;
  return static_cast<size_t>(groups * 2 * K + groups * 8 + kMaxWarps * 4 + KW * 8 + rows * 8);
}

__device__ __forceinline__ void group_sync(int g, int nthreads) {
  if (nthreads == 32) __syncwarp();
  else asm volatile("bar.sync %0, %1;" ::"r"(1 + g), "r"(nthreads) : "memory");
}

// The rows of a block are dealt to G row groups of GW warps (G = the number
// of row slots that fit, GW so that each lane takes a few 8-column vectors
// of a row).  Group g takes the rows g, g + G, ... and streams them through
// its slot.
__global__ void __launch_bounds__(kMaxWarps * 32, 1) xact_rows_kernel(RowActArgs a) {
  extern __shared__ __align__(128) unsigned char sm[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int NT = blockDim.x, NW = NT >> 5;
  const int G = a.groups, GW = NW / G;
  const int K = a.K, M = a.M, R = a.rows_per_block;
  const int nvec = K / 8, KW = (K + 31) / 32;
  const int r0 = static_cast<int>(blockIdx.x) * R;
  const int nr = min(R, M - r0);
  const uint32_t row_bytes = 2u * static_cast<uint32_t>(K);

  uint4* slots = reinterpret_cast<uint4*>(sm);                                            // [G][nvec]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + static_cast<size_t>(G) * row_bytes);  // [G]
  uint32_t* red_s = reinterpret_cast<uint32_t*>(bars + G);                               // [kMaxWarps]
  uint32_t* mask_s = red_s + kMaxWarps;                                                  // [KW]
  int* pre_s = reinterpret_cast<int*>(mask_s + KW);                                      // [KW]
  uint32_t* smax_s = reinterpret_cast<uint32_t*>(pre_s + KW);                            // [R] S_i bits
  uint32_t* redo_s = smax_s + R;                                                         // [R] step-5 marks
  __shared__ uint32_t s_gen;
  __shared__ int s_ok, s_count;
  __shared__ int s_flagged;  // rows of the block flagged so far
  __shared__ int s_marked;   // a row is marked for step 5

  // The GEMM that follows may launch now; its blocks take the SMs this
  // kernel leaves.
  pdl_launch_dependents();
  if (tid == 0) {
    s_gen = *reinterpret_cast<volatile uint32_t*>(a.sync + 2);
    for (int g = 0; g < G; ++g) mbar_init(&bars[g], 1);
    fence_mbar_init();
  }
  for (int w = tid; w < KW; w += NT) mask_s[w] = 0u;
  for (int i = tid; i < R; i += NT) redo_s[i] = 0u;
  if (tid == 0) {
    s_flagged = 0;
    s_marked = 0;
  }
  __syncthreads();

  // ------------------------------------------------------------- phase 1
  const bool all_out = a.thr < 0;  // alpha < 0: every column is an outlier
  const uint32_t thr2 = all_out ? 0u : static_cast<uint32_t>(a.thr) * 0x00010001u;
  const int g = warp / GW, wg = warp - g * GW;  // row group, warp within it
  const int gthreads = GW * 32, gt = wg * 32 + lane;
  const bool leader = gt == 0;
  const int my_rows = nr > g ? (nr - g + G - 1) / G : 0;  // local rows g + j G
  uint4* slot = slots + static_cast<size_t>(g) * nvec;
  uint64_t* bar = &bars[g];
  auto issue = [&](int j) {  // leader: the bulk copy of the group's j-th row into its slot
    const int lr = g + j * G;
    mbar_arrive_expect_tx(bar, row_bytes);
    bulk_load_1d(slot, reinterpret_cast<const unsigned char*>(a.X) + static_cast<size_t>(r0 + lr) * row_bytes,
                 row_bytes, bar);
  };
  // all lanes of the group agree on v (a wait that ran out in one of them)
  auto group_all = [&](bool v) -> bool {
    if (GW == 1) return __all_sync(0xffffffffu, v);
    uint32_t r;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 q, %1, 0;\n bar.red.and.pred p, %2, %3, q;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(v)), "r"(1 + g), "r"(gthreads)
        : "memory");
    return r != 0;
  };
  // (1) waits for the group's j-th row, then flags the columns of its
  //     entries above alpha in the block's bitmask (a branch per vector
  //     that holds one)
  auto land_and_flag = [&](int j) -> bool {
    bool landed = mbar_wait(bar, static_cast<uint32_t>(j & 1), a.timeout_ns, nullptr);
    if (!group_all(landed)) {
      // leave no bulk copy in flight into the slot before the block can exit
      mbar_wait(bar, static_cast<uint32_t>(j & 1), a.timeout_ns, nullptr);
      return false;
    }
#pragma unroll 4
    for (int v = gt; v < nvec; v += gthreads) {
      const uint4 x = slot[v];
      const uint32_t m0 = x.x & 0x7fff7fffu, m1 = x.y & 0x7fff7fffu;
      const uint32_t m2 = x.z & 0x7fff7fffu, m3 = x.w & 0x7fff7fffu;
      const uint32_t f = __vmaxu2(__vmaxu2(m0, m1), __vmaxu2(m2, m3));
      if (all_out || __vcmpgtu2(f, thr2) != 0u) {
        const uint32_t mw[4] = {m0, m1, m2, m3};
        uint32_t fl = 0u;
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const uint32_t big = all_out ? 0xffffffffu : __vcmpgtu2(mw[p], thr2);
          fl |= ((big & 1u) << (2 * p)) | (((big >> 16) & 1u) << (2 * p + 1));
        }
        atomicOr(&mask_s[v >> 2], fl << ((v & 3) * 8));
      }
    }
    return true;
  };
  if (leader && my_rows > 0) issue(0);
  // Rows are quantised as they land, but only once the block has flagged
  // kFirstRows rows (fewer if it has fewer rows or row groups: before the
  // wait ends, only each group's first row can be flagged): the outlier
  // columns then show in the block's bitmask (in the pages' activations an
  // outlier column is large in most rows), so S_i below leaves them out and
  // rarely needs the correction after the barrier.
  const int need_flagged = min(min(nr, G), kFirstRows);
  int ok = 1;
  for (int j = 0; j < my_rows && ok; ++j) {
    const int lr = g + j * G;
    if (!land_and_flag(j)) {
      ok = 0;
      break;
    }
    group_sync(g, gthreads);  // the group's flags are in the bitmask
    if (leader) {
      __threadfence_block();
      atomicAdd(&s_flagged, 1);
    }
    if (j == 0) {  // later rows come after the first kFirstRows anyway
      const uint64_t t0 = global_timer_ns();
      for (uint32_t it = 0; *reinterpret_cast<volatile int*>(&s_flagged) < need_flagged; ++it) {
        if ((it & 15u) == 15u && global_timer_ns() - t0 > a.timeout_ns) {
          ok = 0;
          break;
        }
      }
      __threadfence_block();
      if (!group_all(ok)) {
        ok = 0;
        break;
      }
    }
    // (2) S_i: max |x| over the columns not flagged so far (every entry
    //     above alpha is flagged, by the lane that reads it again here)
    uint32_t rm = 0u;
#pragma unroll 4
    for (int v = gt; v < nvec; v += gthreads) {
      const uint32_t fl = (mask_s[v >> 2] >> ((v & 3) * 8)) & 0xffu;
      rm = masked_absmax2(rm, slot[v], fl);
    }
    uint32_t S = __reduce_max_sync(0xffffffffu, max_pair(rm));
    if (GW > 1) {
      if (lane == 0) red_s[warp] = S;
      group_sync(g, gthreads);
      for (int u = 0; u < GW; ++u) S = max(S, red_s[g * GW + u]);
    }
    const float c = scale_from_absmax_bits(S);
    // (3) the codes of every column with c = 127 / S_i; those of the
    //     outlier columns are set to 0 after the barrier
    int8_t* qrow = a.Xq + static_cast<size_t>(r0 + lr) * K;
#pragma unroll 4
    for (int v = gt; v < nvec; v += gthreads)
      *reinterpret_cast<uint2*>(qrow + static_cast<size_t>(v) * 8) = quant8_fma(slot[v], c);
    if (leader) {
      smax_s[lr] = S;
      a.c_x[r0 + lr] = c;
    }
    group_sync(g, gthreads);  // the group is done with the slot (and with red_s)
    if (leader && j + 1 < my_rows) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      issue(j + 1);
    }
  }

  // the block's outlier bits into the global bitmask of this generation
  ok = __syncthreads_and(ok);
  const uint32_t gen = s_gen;
  uint32_t* gmask = a.omask + static_cast<size_t>(gen & 1u) * KW;
  for (int w = tid; w < KW; w += NT) {
    const uint32_t b = mask_s[w];
    if (b) atomicOr(gmask + w, b);
  }

  // ------------------------------------------------------------- phase 2
  // grid barrier (every block arrives, also after a failed wait above)
  __syncthreads();
  if (tid == 0) {
    uint32_t* arrivals = a.sync + (gen & 1u);
    if (!(a.skip_arrival && blockIdx.x == 0)) red_release_add_gpu(arrivals, 1u);
    int bar_ok = 1;
    if (ld_acquire_gpu_u32(arrivals) < gridDim.x) {
      const uint64_t t0 = global_timer_ns();
      for (uint32_t it = 1; ld_acquire_gpu_u32(arrivals) < gridDim.x; ++it) {
        if ((it & 15u) == 0 && global_timer_ns() - t0 > a.timeout_ns) {
          bar_ok = 0;
          break;
        }
      }
    }
    if (!ok || !bar_ok) atomicOr(a.status, kStatusTimeout);
    s_ok = ok && bar_ok;
  }
  __syncthreads();
  if (!s_ok) return;  // no copy is in flight: every group waited for its last one
  if (blockIdx.x == 0 && tid == 0) {
    // every block has read the generation (before arriving)
    a.sync[(gen + 1u) & 1u] = 0u;
    a.sync[2] = gen + 1u;
  }

  // ------------------------------------------------------------- phase 3
  // the global bitmask; one warp forms the exclusive prefix of its word
  // popcounts (and, in block 0, the index list and the count)
  for (int w = tid; w < KW; w += NT) mask_s[w] = __ldcg(gmask + w);
  __syncthreads();
  if (warp == 0) {
    const int wpl = (KW + 31) / 32;
    const int w0 = min(KW, lane * wpl), w1 = min(KW, w0 + wpl);
    int cnt = 0;
    for (int w = w0; w < w1; ++w) cnt += __popc(mask_s[w]);
    int incl = cnt;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += u;
    }
    int pos = incl - cnt;
    for (int w = w0; w < w1; ++w) {
      pre_s[w] = pos;
      pos += __popc(mask_s[w]);
    }
    if (lane == 31) {
      s_count = incl;
      if (blockIdx.x == 0) *a.count = incl;
    }
  }
  if (blockIdx.x == 0) {
    uint32_t* next = a.omask + static_cast<size_t>((gen + 1u) & 1u) * KW;
    for (int w = tid; w < KW; w += NT) next[w] = 0u;
  }
  __syncthreads();
  // the ascending list of outlier columns, in the (now free) row slots: at
  // most K entries of 2 bytes; block 0 also writes it out as idx
  uint16_t* cols = reinterpret_cast<uint16_t*>(slots);
  for (int w = tid; w < KW; w += NT) {
    uint32_t bits = mask_s[w];
    int o = pre_s[w];
    while (bits) {
      const int col = w * 32 + __ffs(bits) - 1;
      bits &= bits - 1;
      cols[o] = static_cast<uint16_t>(col);
      if (blockIdx.x == 0) a.idx[o] = col;
      ++o;
    }
  }
  __syncthreads();
  // (4) every (outlier, row) pair of the block, rows fastest: gather the
  //     entry, zero its code, and mark the row when the entry is <= alpha
  //     and equal to S_i; four pairs' loads in flight per thread
  const int n_out = s_count;
  const unsigned short* xb = reinterpret_cast<const unsigned short*>(a.X);
  const int pairs = n_out * nr;
  for (int p0 = tid; p0 < pairs; p0 += 4 * NT) {
    unsigned short x[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int p = p0 + u * NT;
      x[u] = 0;
      if (p < pairs) {
        const int o = p / nr, r = p - o * nr;
        x[u] = __ldg(xb + static_cast<size_t>(r0 + r) * K + cols[o]);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int p = p0 + u * NT;
      if (p < pairs) {
        const int o = p / nr, r = p - o * nr;
        a.X_OT[static_cast<size_t>(o) * a.ld_xo + r0 + r] = __ushort_as_half(x[u]);
        a.Xq[static_cast<size_t>(r0 + r) * K + cols[o]] = 0;
        const uint32_t mag = x[u] & 0x7fffu;
        if (!all_out && mag <= static_cast<uint32_t>(a.thr) && mag == smax_s[r]) {
          redo_s[r] = 1u;
          s_marked = 1;
        }
      }
    }
  }
  __syncthreads();
  // (5) marked rows, one at a time with the whole block (a row's vectors
  //     spread over all threads, so that its loads are in flight together;
  //     one warp per row took ~16 us for a row): the exact absmax over the
  //     columns outside O, c_x and the codes again (outlier columns 0)
  for (int lr = 0; s_marked && lr < nr; ++lr) {
    if (smax_s[lr] == 0u || redo_s[lr] == 0u) continue;  // block-uniform
    const uint4* xr = reinterpret_cast<const uint4*>(a.X + static_cast<size_t>(r0 + lr) * K);
    uint32_t m = 0u;
    for (int v = tid; v < nvec; v += NT) {
      const uint32_t fl = (mask_s[v >> 2] >> ((v & 3) * 8)) & 0xffu;
      m = masked_absmax2(m, __ldg(xr + v), fl);
    }
    m = __reduce_max_sync(0xffffffffu, max_pair(m));
    if (lane == 0) red_s[warp] = m;
    __syncthreads();
    uint32_t S2 = 0u;
    for (int u = 0; u < NW; ++u) S2 = max(S2, red_s[u]);
    const float c = scale_from_absmax_bits(S2);
    int8_t* qrow = a.Xq + static_cast<size_t>(r0 + lr) * K;
    for (int v = tid; v < nvec; v += NT) {
      const uint32_t fl = (mask_s[v >> 2] >> ((v & 3) * 8)) & 0xffu;
      uint2 q = quant8_fma(__ldg(xr + v), c);
      q.x &= ~expand_nibble(fl & 0xfu);
      q.y &= ~expand_nibble(fl >> 4);
      *reinterpret_cast<uint2*>(qrow + static_cast<size_t>(v) * 8) = q;
    }
    if (tid == 0) a.c_x[r0 + lr] = c;
    __syncthreads();  // red_s is reused by the next marked row
  }
}

struct Shape {
  int64_t rows;    // per block
  int64_t groups;  // row groups per block: one row slot each
  int64_t gw;      // warps per row group
};

Shape shape_for(int64_t M, int64_t K, int num_sms) {
  Shape s;
  s.rows = (M + num_sms - 1) / num_sms;
  const int64_t KW = (K + 31) / 32;
  const int64_t fixed = KW * 8 + s.rows * 8 + kMaxWarps * 4;
  const int64_t per_group = 2 * K + 8;
  const int64_t fit = static_cast<int64_t>(kRowActSmemMax) > fixed
                          ? (static_cast<int64_t>(kRowActSmemMax) - fixed) / per_group
                          : 0;
  s.groups = std::min<int64_t>({s.rows, static_cast<int64_t>(kMaxGroups), fit});
  // warps per group: about four 8-column vectors per lane and row, within
  // the block's 32 warps
  const int64_t nvec = K / 8;
  s.gw = s.groups > 0 ? std::max<int64_t>(1, std::min<int64_t>(kMaxWarps / s.groups, nvec / 128)) : 1;
  return s;
}

}  // namespace

int half_magnitude_threshold(float alpha) {
  if (alpha < 0.0f) return -1;
  // largest binary16 pattern h in [0, 0x7c00] (0 .. +inf) whose value is <= alpha
  auto value = [](int h) -> double {
    const int e = h >> 10, m = h & 0x3ff;
    if (e == 31) return INFINITY;
    return e == 0 ? std::ldexp(static_cast<double>(m), -24) : std::ldexp(static_cast<double>(1024 + m), e - 25);
  };
  int lo = 0, hi = 0x7c00;
  while (lo < hi) {
    const int mid = (lo + hi + 1) / 2;
    if (value(mid) <= static_cast<double>(alpha)) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

bool row_act_fits(int64_t M, int64_t K, int num_sms) {
  if (M <= 0 || K > kRowActMaxK || num_sms <= 0) return false;
  const Shape s = shape_for(M, K, num_sms);
  return s.rows <= kRowActMaxRows && s.groups >= 1;
}

cudaError_t launch_row_act(const RowActArgs& args, int num_sms, cudaStream_t stream) {
  RowActArgs a = args;
  const Shape s = shape_for(a.M, a.K, num_sms);
  if (s.groups < 1 || s.rows > kRowActMaxRows) return cudaErrorInvalidValue;
  a.rows_per_block = static_cast<int>(s.rows);
  a.groups = static_cast<int>(s.groups);
  static unsigned long long attr_set = 0;  // one bit per device
  int dev = 0;
  cudaGetDevice(&dev);
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_set & bit)) {
    cudaError_t e = cudaFuncSetAttribute(xact_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kRowActSmemMax));
    if (e != cudaSuccess) return e;
    attr_set |= bit;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((a.M + s.rows - 1) / s.rows));
  cfg.blockDim = dim3(static_cast<unsigned>(32 * s.groups * s.gw));
  cfg.dynamicSmemBytes = smem_bytes(s.groups, s.rows, a.K);
  cfg.stream = stream;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeCooperative;  // all blocks resident at once (grid barrier)
  attr.val.cooperative = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, xact_rows_kernel, a);
}

}  // namespace i8mm
