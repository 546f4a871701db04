// Memory-bound passes of the LLM.int8() decomposed matmul on sm_100a:
//   * weight preparation: per-column absmax of W, c_w = 127/absmax, int8
//     codes written transposed (K-major) for the tensor cores;
//   * outlier detection: column maxima of X and the compacted outlier set
//     O = {j : max_i |X[i,j]| > alpha};
//   * row quantisation: per row absmax over the non-outlier columns,
//     c_x = 127/absmax, int8 codes with outlier columns zeroed, and the fp16
//     outlier columns gathered for the GEMM epilogue.
//
// Method: "LLM.int8() — 大模型激活值里藏着几个超大异常通道", 方法1 (one scale
// per row of X and per column of W) and 方法2 (columns with |x| > 6 go to
// fp16); "LLM.int8()" (brain.gartu.xyz), "Seuil de détection α"; the Fig. 2
// caption of the AI 十大核心论文解读 article (split, then scale).
//
// All loads of X and W are 16-byte vectors; |x| is handled as the binary16
// magnitude bits (h & 0x7fff), whose unsigned order equals the order of |x|,
// so maxima are exact and two lanes are compared per instruction (vmax2).
#include "kernels.cuh"

#include <algorithm>

namespace i8mm {
namespace {

__device__ __forceinline__ int8_t quant_rne(float x, float c) {
  // fp32 product rounded once, then round-to-nearest-even, clamped to +-127.
  int q = __float2int_rn(__fmul_rn(x, c));
  q = max(-127, min(127, q));
  return static_cast<int8_t>(q);
}

__device__ __forceinline__ float scale_from_absmax_bits(uint32_t bits) {
  const float a = __half2float(__ushort_as_half(static_cast<unsigned short>(bits)));
  return a == 0.0f ? 0.0f : __fdiv_rn(127.0f, a);
}

__device__ __forceinline__ uint32_t max_pair(uint32_t m) { return max(m & 0xffffu, m >> 16); }

// ------------------------------------------------------------------------
// Weight prep, step 1: column absmax of W[K,N] into colmax_bits[N] (atomicMax
// on the magnitude bits).  Block (32, 8): 32 threads x 8 columns = 256
// columns per block, 8 row lanes; gridDim.y splits K into chunks.
__global__ void __launch_bounds__(256) weight_colmax_kernel(const __half* __restrict__ W, int K, int N,
                                                            int rows_per_chunk, uint32_t* colmax_bits) {
  const int tx = threadIdx.x, ty = threadIdx.y;
  const int col = blockIdx.x * 256 + tx * 8;
  const int r0 = blockIdx.y * rows_per_chunk;
  const int r1 = min(K, r0 + rows_per_chunk);
  uint32_t m[4] = {0, 0, 0, 0};
  if (col < N) {
    for (int r = r0 + ty; r < r1; r += 8) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(W + static_cast<size_t>(r) * N + col));
      m[0] = __vmaxu2(m[0], v.x & 0x7fff7fffu);
      m[1] = __vmaxu2(m[1], v.y & 0x7fff7fffu);
      m[2] = __vmaxu2(m[2], v.z & 0x7fff7fffu);
      m[3] = __vmaxu2(m[3], v.w & 0x7fff7fffu);
    }
  }
  __shared__ uint32_t red[8][32][4];
#pragma unroll
  for (int p = 0; p < 4; ++p) red[ty][tx][p] = m[p];
  __syncthreads();
  if (ty == 0 && col < N) {
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      uint32_t v = red[0][tx][p];
      for (int y = 1; y < 8; ++y) v = __vmaxu2(v, red[y][tx][p]);
      if ((v & 0xffffu) != 0) atomicMax(colmax_bits + col + 2 * p, v & 0xffffu);
      if ((v >> 16) != 0) atomicMax(colmax_bits + col + 2 * p + 1, v >> 16);
    }
  }
}

// Weight prep, step 2: codes of a 128(k) x 128(n) tile, transposed through
// shared memory so that both the fp16 reads (along n) and the int8 writes
// (along k) are 16-byte vectors.  Blocks with blockIdx.y == 0 also write
// c_w and 1/c_w.
__global__ void __launch_bounds__(256) weight_quant_kernel(const __half* __restrict__ W, int K, int N,
                                                           const uint32_t* __restrict__ colmax_bits,
                                                           int8_t* __restrict__ Wq_t, float* __restrict__ c_w,
                                                           float* __restrict__ inv_cw) {
  __shared__ float cs[128];
  __shared__ __align__(16) int8_t tile[128][144];  // [n][k], rows padded to 144 B
  const int tid = threadIdx.x;
  const int n0 = blockIdx.x * 128, k0 = blockIdx.y * 128;
  if (tid < 128) {
    const int n = n0 + tid;
    float c = 0.0f;
    if (n < N) {
      c = scale_from_absmax_bits(colmax_bits[n]);
      if (blockIdx.y == 0) {
        c_w[n] = c;
        inv_cw[n] = c == 0.0f ? 0.0f : __frcp_rn(c);
      }
    }
    cs[tid] = c;
  }
  __syncthreads();
  // 16 threads per k-row (8 columns each), 16 rows per pass, 8 passes.
  const int cg = (tid & 15) * 8;
#pragma unroll 2
  for (int pass = 0; pass < 8; ++pass) {
    const int kl = pass * 16 + (tid >> 4);
    const int k = k0 + kl, n = n0 + cg;
    int8_t q[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (k < K && n < N) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(W + static_cast<size_t>(k) * N + n));
      const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const float2 f = __half22float2(h[p]);
        q[2 * p] = quant_rne(f.x, cs[cg + 2 * p]);
        q[2 * p + 1] = quant_rne(f.y, cs[cg + 2 * p + 1]);
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) tile[cg + e][kl] = q[e];
  }
  __syncthreads();
  // 8 threads x 16 bytes per n-row, 32 rows per pass, 4 passes.
#pragma unroll
  for (int pass = 0; pass < 4; ++pass) {
    const int nl = pass * 32 + (tid >> 3);
    const int kc = (tid & 7) * 16;
    const int n = n0 + nl, k = k0 + kc;
    if (n < N && k < K) {
      *reinterpret_cast<uint4*>(Wq_t + static_cast<size_t>(n) * K + k) =
          *reinterpret_cast<const uint4*>(&tile[nl][kc]);
    }
  }
}

// ------------------------------------------------------------------------
// Outlier detection.  Grid (ceil(K/256), chunks), block (32, 8).  Each block
// reduces a 256-column stripe over one chunk of rows into `partial`.  The
// last block to finish a stripe (ticket) reduces the chunks, writes colmax
// and the stripe's 8 mask words; the last stripe to finish (second ticket)
// compacts the mask into the ascending index list and the count.  Tickets
// are returned to zero by the block that consumed them, so no per-launch
// clearing is needed.
__global__ void __launch_bounds__(256) outlier_detect_kernel(const __half* __restrict__ X, int M, int K,
                                                             float alpha, int rows_per_chunk,
                                                             OutlierScratch s) {
  const int tx = threadIdx.x, ty = threadIdx.y, tid = ty * 32 + tx;
  const int stripe = blockIdx.x;
  const int col = stripe * 256 + tx * 8;
  const int r0 = blockIdx.y * rows_per_chunk;
  const int r1 = min(M, r0 + rows_per_chunk);
  uint32_t m[4] = {0, 0, 0, 0};
  if (col < K) {
    const __half* base = X + col;
    int r = r0 + ty;
    for (; r + 24 < r1; r += 32) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        v[u] = __ldg(reinterpret_cast<const uint4*>(base + static_cast<size_t>(r + 8 * u) * K));
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        m[0] = __vmaxu2(m[0], v[u].x & 0x7fff7fffu);
        m[1] = __vmaxu2(m[1], v[u].y & 0x7fff7fffu);
        m[2] = __vmaxu2(m[2], v[u].z & 0x7fff7fffu);
        m[3] = __vmaxu2(m[3], v[u].w & 0x7fff7fffu);
      }
    }
    for (; r < r1; r += 8) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(base + static_cast<size_t>(r) * K));
      m[0] = __vmaxu2(m[0], v.x & 0x7fff7fffu);
      m[1] = __vmaxu2(m[1], v.y & 0x7fff7fffu);
      m[2] = __vmaxu2(m[2], v.z & 0x7fff7fffu);
      m[3] = __vmaxu2(m[3], v.w & 0x7fff7fffu);
    }
  }
  __shared__ uint32_t red[8][32][4];
  __shared__ unsigned s_last;
  __shared__ int s_scan[8];
#pragma unroll
  for (int p = 0; p < 4; ++p) red[ty][tx][p] = m[p];
  __syncthreads();
  if (ty == 0 && col < K) {
    uint4 out;
    uint32_t* o = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      uint32_t v = red[0][tx][p];
      for (int y = 1; y < 8; ++y) v = __vmaxu2(v, red[y][tx][p]);
      o[p] = v;
    }
    *reinterpret_cast<uint4*>(s.partial + static_cast<size_t>(blockIdx.y) * K + col) = out;
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(s.stripe_ticket + stripe, 1u) == gridDim.y - 1) ? 1u : 0u;
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // Last block of this stripe: reduce the chunks, one column per thread.
  {
    const int c = stripe * 256 + tid;
    uint32_t mx = 0;
    if (c < K) {
      for (int ch = 0; ch < static_cast<int>(gridDim.y); ++ch)
        mx = max(mx, static_cast<uint32_t>(__ldcg(s.partial + static_cast<size_t>(ch) * K + c)));
    }
    const float cm = __half2float(__ushort_as_half(static_cast<unsigned short>(mx)));
    if (c < K) s.colmax[c] = cm;
    const unsigned word = __ballot_sync(0xffffffffu, (c < K) && (cm > alpha));
    if (tx == 0 && c < K) s.mask[c >> 5] = word;
    if (tid == 0) s.stripe_ticket[stripe] = 0;
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(s.all_ticket, 1u) == gridDim.x - 1) ? 1u : 0u;
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // Last stripe overall: compact the bitmask into ascending indices.
  const int nwords = (K + 31) / 32;
  const int wpt = (nwords + 255) / 256;
  const int w0 = min(nwords, tid * wpt), w1 = min(nwords, w0 + wpt);
  int cnt = 0;
  for (int w = w0; w < w1; ++w) cnt += __popc(__ldcg(s.mask + w));
  int incl = cnt;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, d);
    if (tx >= d) incl += v;
  }
  if (tx == 31) s_scan[ty] = incl;
  __syncthreads();
  int before = 0, total = 0;
#pragma unroll
  for (int y = 0; y < 8; ++y) {
    const int v = s_scan[y];
    before += (y < ty) ? v : 0;
    total += v;
  }
  int pos = before + incl - cnt;
  for (int w = w0; w < w1; ++w) {
    uint32_t bits = __ldcg(s.mask + w);
    while (bits) {
      const int b = __ffs(bits) - 1;
      s.idx[pos++] = w * 32 + b;
      bits &= bits - 1;
    }
  }
  if (tid == 0) {
    *s.count = total;
    *s.all_ticket = 0;
  }
}

// ------------------------------------------------------------------------
// Row quantisation: one block per row of X; each thread holds VPT vectors
// of 8 halves in registers between the absmax and the quantise steps.
template <int VPT, int NT>
__global__ void __launch_bounds__(NT) row_quant_kernel(const __half* __restrict__ X, int M, int K,
                                                       const uint32_t* __restrict__ mask,
                                                       const int32_t* __restrict__ idx,
                                                       const int32_t* __restrict__ count,
                                                       int8_t* __restrict__ Xq, float* __restrict__ c_x,
                                                       __half* __restrict__ X_OT) {
  const int row = blockIdx.x, tid = threadIdx.x;
  const int nvec = K / 8;
  const uint4* xr = reinterpret_cast<const uint4*>(X + static_cast<size_t>(row) * K);
  uint4 v[VPT];
  uint32_t fl[VPT];
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int c8 = tid + i * NT;
    fl[i] = 0xffu;
    v[i] = make_uint4(0, 0, 0, 0);
    if (c8 < nvec) {
      v[i] = __ldg(xr + c8);
      fl[i] = (__ldg(mask + (c8 >> 2)) >> ((c8 & 3) * 8)) & 0xffu;
    }
    const uint32_t* w = reinterpret_cast<const uint32_t*>(&v[i]);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const uint32_t keep = (((fl[i] >> (2 * p)) & 1u) ? 0u : 0x0000ffffu) |
                            (((fl[i] >> (2 * p + 1)) & 1u) ? 0u : 0xffff0000u);
      m = __vmaxu2(m, w[p] & 0x7fff7fffu & keep);
    }
  }
  m = max_pair(m);
  m = __reduce_max_sync(0xffffffffu, m);
  __shared__ uint32_t s_red[NT / 32];
  __shared__ float s_c;
  if ((tid & 31) == 0) s_red[tid >> 5] = m;
  __syncthreads();
  if (tid < 32) {
    uint32_t t = tid < NT / 32 ? s_red[tid] : 0u;
    t = __reduce_max_sync(0xffffffffu, t);
    if (tid == 0) {
      const float c = scale_from_absmax_bits(t);
      s_c = c;
      c_x[row] = c;
    }
  }
  __syncthreads();
  const float c = s_c;
  int8_t* qr = Xq + static_cast<size_t>(row) * K;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int c8 = tid + i * NT;
    if (c8 < nvec) {
      const __half2* h = reinterpret_cast<const __half2*>(&v[i]);
      uint32_t lo = 0, hi = 0;
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const float2 f = __half22float2(h[p]);
        const uint32_t a = ((fl[i] >> (2 * p)) & 1u) ? 0u : static_cast<uint8_t>(quant_rne(f.x, c));
        const uint32_t b = ((fl[i] >> (2 * p + 1)) & 1u) ? 0u : static_cast<uint8_t>(quant_rne(f.y, c));
        const uint32_t pair = a | (b << 8);
        if (p < 2) lo |= pair << (16 * p);
        else hi |= pair << (16 * (p - 2));
      }
      *reinterpret_cast<uint2*>(qr + c8 * 8) = make_uint2(lo, hi);
    }
  }
  const int cnt = *count;
  for (int o = tid; o < cnt; o += NT)
    X_OT[static_cast<size_t>(o) * M + row] = X[static_cast<size_t>(row) * K + idx[o]];
}

template <int VPT, int NT>
cudaError_t launch_row_quant_t(const __half* X, int64_t M, int64_t K, const OutlierScratch& s, int8_t* Xq,
                               float* c_x, __half* X_OT, cudaStream_t stream) {
  row_quant_kernel<VPT, NT><<<static_cast<unsigned>(M), NT, 0, stream>>>(
      X, static_cast<int>(M), static_cast<int>(K), s.mask, s.idx, s.count, Xq, c_x, X_OT);
  return cudaGetLastError();
}

}  // namespace

// ------------------------------------------------------------------------
cudaError_t launch_weight_prep(const __half* W, int64_t K, int64_t N, uint32_t* colmax_bits, int8_t* Wq_t,
                               float* c_w, float* inv_cw, int num_sms, cudaStream_t stream) {
  cudaError_t e = cudaMemsetAsync(colmax_bits, 0, static_cast<size_t>(N) * sizeof(uint32_t), stream);
  if (e != cudaSuccess) return e;
  const int stripes = static_cast<int>((N + 255) / 256);
  int chunks = std::max(1, (4 * num_sms + stripes - 1) / stripes);
  chunks = static_cast<int>(std::min<int64_t>(chunks, (K + 7) / 8));
  const int rows_per_chunk = static_cast<int>((K + chunks - 1) / chunks);
  chunks = static_cast<int>((K + rows_per_chunk - 1) / rows_per_chunk);
  weight_colmax_kernel<<<dim3(stripes, chunks), dim3(32, 8), 0, stream>>>(
      W, static_cast<int>(K), static_cast<int>(N), rows_per_chunk, colmax_bits);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  weight_quant_kernel<<<dim3(static_cast<unsigned>((N + 127) / 128), static_cast<unsigned>((K + 127) / 128)),
                        256, 0, stream>>>(W, static_cast<int>(K), static_cast<int>(N), colmax_bits, Wq_t,
                                          c_w, inv_cw);
  return cudaGetLastError();
}

namespace {
int64_t chunk_target(int64_t M, int64_t K, int num_sms) {
  const int64_t stripes = (K + 255) / 256;
  const int64_t chunks = std::max<int64_t>(1, (4 * num_sms + stripes - 1) / stripes);
  return std::max<int64_t>(1, std::min<int64_t>(chunks, (M + 7) / 8));
}
}  // namespace

int outlier_row_chunks(int64_t M, int64_t K, int num_sms) {
  const int64_t chunks = chunk_target(M, K, num_sms);
  const int64_t rows_per_chunk = (M + chunks - 1) / chunks;
  return static_cast<int>((M + rows_per_chunk - 1) / rows_per_chunk);
}

int outlier_row_chunks_bound(int64_t M, int64_t K, int num_sms) {
  // non-decreasing in M and >= outlier_row_chunks(M', K) for every M' <= M
  return static_cast<int>(chunk_target(M, K, num_sms));
}

cudaError_t launch_outlier_detect(const __half* X, int64_t M, int64_t K, float alpha, const OutlierScratch& s,
                                  int num_sms, cudaStream_t stream) {
  const int stripes = static_cast<int>((K + 255) / 256);
  const int chunks = outlier_row_chunks(M, K, num_sms);
  const int rows_per_chunk = static_cast<int>((M + chunks - 1) / chunks);
  outlier_detect_kernel<<<dim3(stripes, chunks), dim3(32, 8), 0, stream>>>(
      X, static_cast<int>(M), static_cast<int>(K), alpha, rows_per_chunk, s);
  return cudaGetLastError();
}

cudaError_t launch_row_quant(const __half* X, int64_t M, int64_t K, const OutlierScratch& s, int8_t* Xq,
                             float* c_x, __half* X_OT, cudaStream_t stream) {
  const int64_t nvec = K / 8;
  if (nvec <= 256 * 1) return launch_row_quant_t<1, 256>(X, M, K, s, Xq, c_x, X_OT, stream);
  if (nvec <= 256 * 2) return launch_row_quant_t<2, 256>(X, M, K, s, Xq, c_x, X_OT, stream);
  if (nvec <= 256 * 4) return launch_row_quant_t<4, 256>(X, M, K, s, Xq, c_x, X_OT, stream);
  if (nvec <= 256 * 8) return launch_row_quant_t<8, 256>(X, M, K, s, Xq, c_x, X_OT, stream);
  if (nvec <= 256 * 16) return launch_row_quant_t<16, 256>(X, M, K, s, Xq, c_x, X_OT, stream);
  if (nvec <= 512 * 16) return launch_row_quant_t<16, 512>(X, M, K, s, Xq, c_x, X_OT, stream);
  return cudaErrorInvalidValue;
}

}  // namespace i8mm
