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
// All loads of X and W are 16-byte vectors; maxima are taken on the binary16
// magnitude bits (actq.cuh).
#include "actq.cuh"
#include "kernels.cuh"

#include <algorithm>

namespace i8mm {
namespace {

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
// shared memory, written to the K-blocked layout Wb[kb][n][0..128): the tile
// is one contiguous 16 KB block (codes beyond K are 0).  Blocks with
// blockIdx.y == 0 also write c_w and 1/c_w.
__global__ void __launch_bounds__(256) weight_quant_kernel(const __half* __restrict__ W, int K, int N,
                                                           const uint32_t* __restrict__ colmax_bits,
                                                           int8_t* __restrict__ Wb, int N_pad,
                                                           float* __restrict__ c_w, float* __restrict__ inv_cw) {
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
  // 8 threads x 16 bytes per n-row, 32 rows per pass, 4 passes; the block
  // writes 16 KB of consecutive memory.
  int8_t* dst = Wb + (static_cast<size_t>(blockIdx.y) * N_pad + n0) * 128;
#pragma unroll
  for (int pass = 0; pass < 4; ++pass) {
    const int nl = pass * 32 + (tid >> 3);
    const int kc = (tid & 7) * 16;
    if (n0 + nl < N)
      *reinterpret_cast<uint4*>(dst + nl * 128 + kc) = *reinterpret_cast<const uint4*>(&tile[nl][kc]);
  }
}

// ------------------------------------------------------------------------
// Outlier detection.  ceil(K/256) * ceil(M/64) blocks of (32, 8) threads: a
// block covers a 256-column stripe of a 64-row chunk; thread (tx, ty) reads the
// 8 columns tx*8.. of rows ty, ty+8, .., ty+56 with all 8 loads in flight.
// Column maxima of the chunk are folded into colkey with one 64-bit
// atomicMax per column; the key's high bits hold the launch epoch, so values
// left by earlier launches always lose.  The last block to finish (ticket)
// reads colkey and writes colmax, the outlier bitmask, the per-word prefix
// of its popcounts, the ascending index list and the count, then advances
// the epoch and returns the ticket to zero.
constexpr int kDetectRowsPerThread = 8;
constexpr int kDetectRowsPerBlock = 8 * kDetectRowsPerThread;

__global__ void __launch_bounds__(256) outlier_detect_kernel(const __half* __restrict__ X, int M, int K,
                                                             float alpha, OutlierScratch s) {
  const int tx = threadIdx.x, ty = threadIdx.y, tid = ty * 32 + tx;
  const int stripes = (K + 255) / 256;
  const int col = (static_cast<int>(blockIdx.x) % stripes) * 256 + tx * 8;
  const int r0 = (static_cast<int>(blockIdx.x) / stripes) * kDetectRowsPerBlock;
  const unsigned long long epoch = __ldcg(s.epoch);
  uint32_t m[4] = {0, 0, 0, 0};
  if (col < K) {
    uint4 v[kDetectRowsPerThread];
#pragma unroll
    for (int u = 0; u < kDetectRowsPerThread; ++u) {
      const int r = r0 + ty + 8 * u;
      v[u] = r < M ? __ldg(reinterpret_cast<const uint4*>(X + static_cast<size_t>(r) * K + col))
                   : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kDetectRowsPerThread; ++u) {
      m[0] = __vmaxu2(m[0], v[u].x & 0x7fff7fffu);
      m[1] = __vmaxu2(m[1], v[u].y & 0x7fff7fffu);
      m[2] = __vmaxu2(m[2], v[u].z & 0x7fff7fffu);
      m[3] = __vmaxu2(m[3], v[u].w & 0x7fff7fffu);
    }
  }
  __shared__ uint16_t red[8][256];  // [row lane][column of the stripe]
  __shared__ unsigned s_last;
  __shared__ int s_words[2048];       // popcount per mask word, then its prefix
  __shared__ int s_scan[8];
  {
    uint4 mv = make_uint4(m[0], m[1], m[2], m[3]);
    *reinterpret_cast<uint4*>(&red[ty][tx * 8]) = mv;
  }
  __syncthreads();
  {
    // thread tid owns column tid of the stripe: one atomic per column
    const int c = (static_cast<int>(blockIdx.x) % stripes) * 256 + tid;
    if (c < K) {
      uint32_t v = red[0][tid];
#pragma unroll
      for (int y = 1; y < 8; ++y) v = max(v, static_cast<uint32_t>(red[y][tid]));
      atomicMax(s.colkey + c, (epoch << 16) | v);
      __threadfence();  // the atomic is ordered before the ticket below
    }
  }
  pdl_launch_dependents();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(s.ticket, 1u) == gridDim.x - 1) ? 1u : 0u;
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // Last block: column maxima, bitmask and word popcounts, 256 columns per
  // sweep with 16 sweeps' loads in flight.
  const int nwords = (K + 31) / 32;
  for (int base = 0; base < K; base += 16 * 256) {
    unsigned long long key[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int c = base + u * 256 + tid;
      key[u] = c < K ? __ldcg(s.colkey + c) : 0ull;
    }
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int c = base + u * 256 + tid;
      const float cm = __half2float(__ushort_as_half(static_cast<unsigned short>(key[u] & 0xffffu)));
      if (c < K) s.colmax[c] = cm;
      const unsigned word = __ballot_sync(0xffffffffu, c < K && cm > alpha);
      const int w = (base + u * 256) / 32 + ty;
      if (tx == 0 && w < nwords) {
        s.mask[w] = word;
        s_words[w] = __popc(word);
      }
    }
  }
  __syncthreads();
  // exclusive prefix over the words: thread t takes a run of words
  const int wpt = (nwords + 255) / 256;
  const int w0 = min(nwords, tid * wpt), w1 = min(nwords, w0 + wpt);
  int cnt = 0;
  for (int w = w0; w < w1; ++w) cnt += s_words[w];
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
    s.pre[w] = pos;
    uint32_t bits = __ldcg(s.mask + w);
    while (bits) {
      const int b = __ffs(bits) - 1;
      s.idx[pos++] = w * 32 + b;
      bits &= bits - 1;
    }
  }
  if (tid == 0) {
    *s.count = total;
    *s.epoch = epoch + 1;
    *s.ticket = 0;
  }
}

// ------------------------------------------------------------------------
// Row quantisation: one block per row of X; each thread holds VPT vectors
// of 8 halves in registers between the absmax and the quantise steps.  The
// slot of an outlier entry is pre[word] + (set bits below it in its word).
template <int VPT, int NT>
__global__ void __launch_bounds__(NT) row_quant_kernel(const __half* __restrict__ X, int M, int K,
                                                       const uint32_t* __restrict__ mask,
                                                       const int32_t* __restrict__ pre,
                                                       int8_t* __restrict__ Xq, float* __restrict__ c_x,
                                                       __half* __restrict__ X_OT, int ld_xo) {
  const int row = blockIdx.x, tid = threadIdx.x;
  const int nvec = K / 8;
  const uint4* xr = reinterpret_cast<const uint4*>(X + static_cast<size_t>(row) * K);
  uint4 v[VPT];
  uint32_t fl[VPT];
  // X is an input of the forward, not a result of the detection pass: load
  // the row before waiting for that pass to finish.
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int c8 = tid + i * NT;
    v[i] = c8 < nvec ? __ldg(xr + c8) : make_uint4(0, 0, 0, 0);
  }
  pdl_wait();
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int c8 = tid + i * NT;
    fl[i] = c8 < nvec ? (__ldcg(mask + (c8 >> 2)) >> ((c8 & 3) * 8)) & 0xffu : 0xffu;
    m = masked_absmax2(m, v[i], fl[i]);
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
      uint2 q = quant8(v[i], c);
      if (fl[i]) {  // outlier columns: code 0, and the fp16 value goes to its slot
        q.x &= ~expand_nibble(fl[i] & 0xfu);
        q.y &= ~expand_nibble(fl[i] >> 4);
        const int w = c8 >> 2, sh = (c8 & 3) * 8;
        int o = __ldcg(pre + w) + __popc(__ldcg(mask + w) & ((1u << sh) - 1u));
        const unsigned short* hs = reinterpret_cast<const unsigned short*>(&v[i]);
#pragma unroll
        for (int e = 0; e < 8; ++e)
          if ((fl[i] >> e) & 1u) {
            X_OT[static_cast<size_t>(o) * ld_xo + row] = __ushort_as_half(hs[e]);
            ++o;
          }
      }
      *reinterpret_cast<uint2*>(qr + c8 * 8) = q;
    }
  }
  pdl_launch_dependents();
}

template <int VPT, int NT>
cudaError_t launch_row_quant_t(const __half* X, int64_t M, int64_t K, const OutlierScratch& s, int8_t* Xq,
                               float* c_x, __half* X_OT, int64_t ld_xo, bool pdl, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(M));
  cfg.blockDim = dim3(NT);
  cfg.stream = stream;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, row_quant_kernel<VPT, NT>, X, static_cast<int>(M), static_cast<int>(K),
                            static_cast<const uint32_t*>(s.mask), static_cast<const int32_t*>(s.pre), Xq, c_x,
                            X_OT, static_cast<int>(ld_xo));
}

}  // namespace

// ------------------------------------------------------------------------
cudaError_t launch_weight_prep(const __half* W, int64_t K, int64_t N, uint32_t* colmax_bits, int8_t* Wb,
                               int64_t N_pad, float* c_w, float* inv_cw, int num_sms, cudaStream_t stream) {
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
                        256, 0, stream>>>(W, static_cast<int>(K), static_cast<int>(N), colmax_bits, Wb,
                                          static_cast<int>(N_pad), c_w, inv_cw);
  return cudaGetLastError();
}

cudaError_t launch_outlier_detect(const __half* X, int64_t M, int64_t K, float alpha, const OutlierScratch& s,
                                  cudaStream_t stream) {
  const int64_t stripes = (K + 255) / 256;
  const int64_t chunks = (M + kDetectRowsPerBlock - 1) / kDetectRowsPerBlock;
  outlier_detect_kernel<<<static_cast<unsigned>(stripes * chunks), dim3(32, 8), 0, stream>>>(
      X, static_cast<int>(M), static_cast<int>(K), alpha, s);
  return cudaGetLastError();
}

cudaError_t launch_row_quant(const __half* X, int64_t M, int64_t K, const OutlierScratch& s, int8_t* Xq,
                             float* c_x, __half* X_OT, int64_t ld_xo, bool pdl, cudaStream_t stream) {
  // 128 threads per row up to K = 16384, then 256 and 512; each thread
  // keeps VPT vectors of 8 halves of its row in registers.
  const int64_t nvec = K / 8;
#define I8MM_ROWQ(V, T) \
  if (nvec <= int64_t(V) * (T)) return launch_row_quant_t<V, T>(X, M, K, s, Xq, c_x, X_OT, ld_xo, pdl, stream)
  I8MM_ROWQ(1, 128);
  I8MM_ROWQ(2, 128);
  I8MM_ROWQ(3, 128);
  I8MM_ROWQ(4, 128);
  I8MM_ROWQ(6, 128);
  I8MM_ROWQ(8, 128);
  I8MM_ROWQ(12, 128);
  I8MM_ROWQ(16, 128);
  I8MM_ROWQ(16, 256);
  I8MM_ROWQ(16, 512);
#undef I8MM_ROWQ
  return cudaErrorInvalidValue;
}

}  // namespace i8mm
