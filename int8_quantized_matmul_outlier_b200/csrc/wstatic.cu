// Per-forward gather of the outlier weight rows for the memory-saving
// prepared weight (declared in wstatic.cuh, which states the method).
#include "actq.cuh"
#include "wstatic.cuh"

namespace i8mm {
namespace {

constexpr int G_THREADS = 256;

__global__ void __launch_bounds__(G_THREADS) gather_outlier_rows_kernel(const GatherArgs a) {
  pdl_wait();  // idx and count come from the activation pass
  pdl_launch_dependents();
  const int cnt = *a.count;
  const int cw = min(cnt, a.cap);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    *a.count_w = cw;
    if (cnt > a.cap) atomicOr(a.status, kStatusOutlierCap);
  }
  const int nv = a.N / 8;  // 8 halves (16 bytes) per item
  const long long total = static_cast<long long>(cw) * nv;
  for (long long e = static_cast<long long>(blockIdx.x) * G_THREADS + threadIdx.x; e < total;
       e += static_cast<long long>(gridDim.x) * G_THREADS) {
    const int o = static_cast<int>(e / nv);
    const int n0 = static_cast<int>(e - static_cast<long long>(o) * nv) * 8;
    const int k = __ldg(a.idx + o);
    const int r = __ldg(a.wmap + k);
    uint4 v;
    if (r >= 0) {
      v = __ldg(reinterpret_cast<const uint4*>(a.Wc + static_cast<size_t>(r) * a.N + n0));
    } else {
      // not a stored dimension: w = q / c_w from the codes, fp32, then fp16
      const int8_t* codes = a.Wb + (static_cast<size_t>(k >> 7) * a.N_pad + n0) * 128 + (k & 127);
      __half h[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float q = static_cast<float>(__ldg(codes + static_cast<size_t>(j) * 128));
        h[j] = __float2half_rn(__fmul_rn(q, __ldg(a.inv_cw + n0 + j)));
      }
      v = *reinterpret_cast<const uint4*>(h);
    }
    *reinterpret_cast<uint4*>(a.WO + static_cast<size_t>(o) * a.N + n0) = v;
  }
}

}  // namespace

cudaError_t launch_gather_outlier_rows(const GatherArgs& a, int num_sms, bool pdl, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(num_sms);
  cfg.blockDim = dim3(G_THREADS);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, gather_outlier_rows_kernel, a);
}

}  // namespace i8mm
