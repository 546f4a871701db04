// Activation pass for few tokens (M <= 64) in one kernel on one thread-block
// cluster: outlier-column detection, vector-wise row quantisation and the
// fp16 outlier gather.
//
//   O      = { j : max_i |X[i,j]| > alpha }                        (ascending)
//   c_x[i] = 127 / max_{j not in O} |X[i,j]|,  Xq = rne(X c_x), 0 on O
//   X_OT[o][i] = X[i, O_o]
//
// Method: "LLM.int8() — 大模型激活值里藏着几个超大异常通道", 方法1 and 方法2;
// "LLM.int8()" (brain.gartu.xyz), "Seuil de détection α"; the Fig. 2 caption
// of the AI 十大核心论文解读 article (split, then scale).
//
// The cluster has 16 blocks; block `rank` owns a slice of the K columns (a
// multiple of 32 columns) for all M rows, copied once into its shared memory
// with every load in flight; all later phases read shared memory, and the
// blocks exchange through distributed shared memory:
//   1. column maxima of the slice (thread per 8-column vector), outlier flags,
//      the slice's bitmask words, their prefix and outlier count, and each
//      row's maximum over the slice's non-outlier columns; cluster barrier
//   2. the slice's global outlier offset and the whole count (from every
//      block's count), each row's scale (from every block's row maximum),
//      the ascending index list;
//   3. the codes and the outlier entries of the slice;    cluster barrier
// The forward uses this kernel while the slice fits (M <= 64 and
// M * K/16 * 2 bytes within kSmallActSmemMax).
#include "actq.cuh"
#include "kernels.cuh"

#include <cooperative_groups.h>

namespace cg = cooperative_groups;

namespace i8mm {
namespace {

constexpr int NT = 256;

__global__ void __launch_bounds__(NT) xact_small_kernel(SmallActArgs a) {
  cg::cluster_group cluster = cg::this_cluster();
  const int CL = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int M = a.M, K = a.K, nvec = K / 8;
  // vectors per block, a multiple of 4 so that a 32-column mask word never
  // straddles two blocks
  const int vpb = ((nvec + CL - 1) / CL + 3) / 4 * 4;
  const int v0 = min(nvec, rank * vpb), v1 = min(nvec, v0 + vpb);
  const int nv = v1 - v0;
  const int nw = (nv + 3) / 4;  // mask words of this slice

  // the decode GEMM may start its prologue and weight prefetch right away
  pdl_launch_dependents();

  extern __shared__ uint4 dsm[];
  uint4* xs = dsm;                                               // [M][vpb] the slice of X
  uint4* red_s = xs + M * vpb;                                   // [8][vpb] partial column maxima
  uint8_t* flags = reinterpret_cast<uint8_t*>(red_s + 8 * vpb);   // [vpb]
  uint32_t* mask_s = reinterpret_cast<uint32_t*>(flags + vpb);    // [vpb/4]
  int* wpre_s = reinterpret_cast<int*>(mask_s + vpb / 4);         // [vpb/4]
  __shared__ int s_count;    // outliers in this slice (read by the other blocks)
  __shared__ int s_offset;   // outliers in the lower-rank slices
  __shared__ uint32_t s_rowmax[kDecodeMaxM];  // per row, over this slice's non-outlier columns
  __shared__ float s_c[kDecodeMaxM];
  __shared__ int s_scan[NT / 32];

  // ------------------------------------------------------------- phase 0
  // the slice into shared memory: 8 independent loads in flight per thread
  {
    const uint4* xg = reinterpret_cast<const uint4*>(a.X) + v0;
    const int items = M * nv;
    for (int base = 0; base < items; base += 8 * NT) {
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int it = base + u * NT + tid;
        v[u] = it < items ? __ldg(xg + static_cast<size_t>(it / nv) * nvec + it % nv) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int it = base + u * NT + tid;
        if (it < items) xs[(it / nv) * vpb + it % nv] = v[u];
      }
    }
  }
  __syncthreads();

  // ------------------------------------------------------------- phase 1
  // column maxima: G groups of threads split the rows of each vector
  {
    const int G = max(1, min(NT / max(nv, 1), 8));
    const int g = tid / nv, vlg = tid % nv;
    if (nv > 0 && g < G) {
      for (int vl = vlg; vl < nv; vl += NT) {  // (only loops when nv > NT)
        uint32_t m0 = 0, m1 = 0, m2 = 0, m3 = 0;
        for (int r = g; r < M; r += G) {
          const uint4 v = xs[r * vpb + vl];
          m0 = __vmaxu2(m0, v.x & 0x7fff7fffu);
          m1 = __vmaxu2(m1, v.y & 0x7fff7fffu);
          m2 = __vmaxu2(m2, v.z & 0x7fff7fffu);
          m3 = __vmaxu2(m3, v.w & 0x7fff7fffu);
        }
        red_s[g * vpb + vl] = make_uint4(m0, m1, m2, m3);
      }
    }
    __syncthreads();
    for (int vl = tid; vl < nv; vl += NT) {
      uint4 t = red_s[vl];
      for (int gg = 1; gg < G; ++gg) {
        const uint4 u = red_s[gg * vpb + vl];
        t.x = __vmaxu2(t.x, u.x);
        t.y = __vmaxu2(t.y, u.y);
        t.z = __vmaxu2(t.z, u.z);
        t.w = __vmaxu2(t.w, u.w);
      }
      const unsigned short* hs = reinterpret_cast<const unsigned short*>(&t);
      uint32_t fl = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float cm = __half2float(__ushort_as_half(hs[e]));
        a.colmax[(v0 + vl) * 8 + e] = cm;
        fl |= (cm > a.alpha ? 1u : 0u) << e;
      }
      flags[vl] = static_cast<uint8_t>(fl);
    }
  }
  for (int vl = nv + tid; vl < nw * 4; vl += NT) flags[vl] = 0;  // pad the last word
  __syncthreads();
  {
    // words of the slice, their exclusive prefix and the slice's count
    const int wpt = (nw + NT - 1) / NT;
    const int w0 = min(nw, tid * wpt), w1 = min(nw, w0 + wpt);
    int cnt = 0;
    for (int w = w0; w < w1; ++w) {
      const uint32_t bits = flags[4 * w] | (flags[4 * w + 1] << 8) | (flags[4 * w + 2] << 16) |
                            (static_cast<uint32_t>(flags[4 * w + 3]) << 24);
      mask_s[w] = bits;
      cnt += __popc(bits);
    }
    int incl = cnt;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += v;
    }
    if (lane == 31) s_scan[warp] = incl;
    __syncthreads();
    int before = 0, total = 0;
#pragma unroll
    for (int y = 0; y < NT / 32; ++y) {
      before += (y < warp) ? s_scan[y] : 0;
      total += s_scan[y];
    }
    int pos = before + incl - cnt;
    for (int w = w0; w < w1; ++w) {
      wpre_s[w] = pos;
      pos += __popc(mask_s[w]);
    }
    if (tid == 0) s_count = total;
  }
  // row maxima over this slice's non-outlier columns: warp w takes rows w, w+8, ..
  for (int r = warp; r < M; r += NT / 32) {
    uint32_t mx = 0;
    for (int vl = lane; vl < nv; vl += 32) mx = masked_absmax2(mx, xs[r * vpb + vl], flags[vl]);
    mx = max(mx & 0xffffu, mx >> 16);
    mx = __reduce_max_sync(0xffffffffu, mx);
    if (lane == 0) s_rowmax[r] = mx;
  }
  cluster.sync();

  // ------------------------------------------------------------- phase 2
  // slice offset and the whole outlier count from every block's count; each
  // row's scale from every block's row maximum
  if (warp == 0) {
    const int c = lane < CL ? *cluster.map_shared_rank(&s_count, lane) : 0;
    const int below = __reduce_add_sync(0xffffffffu, lane < rank ? c : 0);
    const int all = __reduce_add_sync(0xffffffffu, c);
    if (lane == 0) {
      s_offset = below;
      if (rank == CL - 1) *a.count = all;
    }
  }
  for (int r = warp; r < M; r += NT / 32) {
    uint32_t m = lane < CL ? *cluster.map_shared_rank(&s_rowmax[r], lane) : 0u;
    m = __reduce_max_sync(0xffffffffu, m);
    const float c = scale_from_absmax_bits(m);
    if (lane == 0) {
      s_c[r] = c;
      if (rank == 0) a.c_x[r] = c;
    }
  }
  __syncthreads();
  const int offset = s_offset;
  for (int w = tid; w < nw; w += NT) {
    uint32_t bits = mask_s[w];
    int pos = offset + wpre_s[w];
    while (bits) {
      const int b = __ffs(bits) - 1;
      a.idx[pos++] = (v0 + 4 * w) * 8 + b;
      bits &= bits - 1;
    }
  }

  // ------------------------------------------------------------- phase 3
  // codes: one (row, vector) item per thread, consecutive threads on
  // consecutive vectors of a row (coalesced stores)
  for (int it = tid; it < M * nv; it += NT) {
    const int r = it / nv, vl = it % nv;
    const uint32_t fl = flags[vl];
    const uint4 v = xs[r * vpb + vl];
    uint2 q = quant8(v, s_c[r]);
    if (fl) {
      q.x &= ~expand_nibble(fl & 0xfu);
      q.y &= ~expand_nibble(fl >> 4);
      const int w = vl >> 2, sh = (vl & 3) * 8;
      int o = offset + wpre_s[w] + __popc(mask_s[w] & ((1u << sh) - 1u));
      const unsigned short* hs = reinterpret_cast<const unsigned short*>(&v);
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if ((fl >> e) & 1u) {
          a.X_OT[static_cast<size_t>(o) * a.ld_xo + r] = __ushort_as_half(hs[e]);
          ++o;
        }
    }
    *reinterpret_cast<uint2*>(a.Xq + static_cast<size_t>(r) * K + static_cast<size_t>(v0 + vl) * 8) = q;
  }
  cluster.sync();  // no block leaves while another may still read its shared memory
}

}  // namespace

namespace {
constexpr int kCluster = 16;

size_t smem_for(int64_t M, int64_t K) {
  const int64_t nvec = K / 8;
  const int64_t vpb = ((nvec + kCluster - 1) / kCluster + 3) / 4 * 4;
  return static_cast<size_t>((M + 8) * vpb * 16 + vpb + (vpb / 4) * 8);
}
}  // namespace

bool small_act_fits(int64_t M, int64_t K) { return M <= kDecodeMaxM && smem_for(M, K) <= kSmallActSmemMax; }

cudaError_t launch_small_act(const SmallActArgs& a, cudaStream_t stream) {
  static unsigned long long attr_set = 0;  // one bit per device
  int dev = 0;
  cudaGetDevice(&dev);
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_set & bit)) {
    cudaError_t e = cudaFuncSetAttribute(xact_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kSmallActSmemMax));
    if (e == cudaSuccess) e = cudaFuncSetAttribute(xact_small_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    attr_set |= bit;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kCluster);
  cfg.blockDim = dim3(NT);
  cfg.dynamicSmemBytes = smem_for(a.M, a.K);
  cfg.stream = stream;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = kCluster;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, xact_small_kernel, a);
}

}  // namespace i8mm
