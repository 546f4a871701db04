// Memory-saving prepared weight: the fp16 rows of W are kept only for a
// calibrated set of input dimensions instead of borrowing all of W.
//
// Method: "LLM.int8() — 大模型激活值里藏着几个超大异常通道" (the outlier
// dimensions are systematic: a few fixed feature dimensions carry them in
// every layer) and 方法2 of the same page (only those dimensions take the fp16
// path, a small fraction of the weight).  The pages do not say what to do
// with an outlier column outside a stored set; here its weight row is
// rebuilt from the int8 codes, w = q / c_w, in fp32 and rounded to fp16.
//
// Both GEMM kernels address the weight rows of the outlier product as
// W[idx[o] * N + n] and use idx for nothing else.  Per forward, a small
// kernel writes this forward's outlier rows, in the order of idx, into a
// handle-owned buffer WO, and the GEMMs are given W = WO and idx = 0, 1, 2,
// ...: the GEMM kernels are the ones of the borrowed-weight path.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace i8mm {

// Status bit: a forward found more outlier columns than the static weight's
// capacity; the outlier product of the columns past it was left out.
constexpr int kStatusOutlierCap = 2;

struct GatherArgs {
  const int32_t* idx;    // [K] ascending outlier columns (from the activation pass)
  const int32_t* count;  // [1] |O|
  const int32_t* wmap;   // [K] slot of input dimension k in Wc, or -1
  const __half* Wc;      // [R][N] the stored fp16 rows of W
  const int8_t* Wb;      // K-blocked int8 codes [K/128][N_pad][128]
  const float* inv_cw;   // [N] 1/c_w (0 for an all-zero column)
  int N, N_pad;
  int cap;               // rows WO holds
  __half* WO;            // [cap][N] this forward's outlier rows, in the order of idx
  int32_t* count_w;      // [1] min(|O|, cap): the count the GEMM uses
  int* status;
};

// One launch per forward, after the activation pass (a programmatic dependent
// of it with `pdl`); the GEMM follows as a programmatic dependent of this one.
cudaError_t launch_gather_outlier_rows(const GatherArgs& a, int num_sms, bool pdl, cudaStream_t stream);

}  // namespace i8mm
