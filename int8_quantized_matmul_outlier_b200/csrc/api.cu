// C ABI of libint8mm.so (declared in include/int8mm.h): weight handles, the
// per-forward workspace, TMA descriptors, argument checks and the launch
// sequence of the decomposed int8 matmul.
#include "int8mm.h"
#include "kernels.cuh"
#include "selftest.cuh"
#include "wstatic.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <functional>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <unordered_set>
#include <vector>

using namespace i8mm;

// Row chunks of the host-buffer forward's prefill GEMM (Y of one chunk is
// copied out while the next computes).
constexpr int kHostChunks = 4;

struct int8mm_weight {
  int device = 0;
  int num_sms = 148;
  int64_t K = 0, N = 0;
  const __half* W = nullptr;  // borrowed fp16 weight [K, N] (nullptr for a static weight)
  int64_t N_pad = 0;          // N rounded up to kWeightRowPad
  int8_t* Wb = nullptr;       // [K/128][N_pad][128] int8 codes, K-blocked
  float* c_w = nullptr;       // [N]
  float* inv_cw = nullptr;    // [N]
  uint32_t* colmax_bits = nullptr;  // [N] prep scratch
  CUtensorMap tmW128;  // Wb, 128-row boxes (operand B of the prefill GEMM, A of the decode GEMM)
  // decode (M <= kDecodeMaxM) scratch: int32 partial sums and per-n-block tickets
  int32_t* part = nullptr;
  unsigned* dticket = nullptr;
  // prefill split-K scratch: partial tiles and per-(tile, CTA, half) tickets
  int split_override = 0;        // 0: automatic
  int32_t* sk_ws = nullptr;
  size_t sk_ws_elems = 0;
  uint32_t* sk_ticket = nullptr;
  size_t sk_ticket_n = 0;
  // fixed-size scratch of the outlier pass
  unsigned long long* colkey = nullptr;  // [K]
  unsigned long long* epoch = nullptr;   // [1]
  unsigned* ticket = nullptr;            // [1]
  uint32_t* mask = nullptr;
  int32_t* pre = nullptr;
  // single-launch activation pass: two bitmasks (by generation parity) and
  // the grid barrier's arrival counter and generation
  uint32_t* omask = nullptr;  // [2][ceil(K/32)]
  uint32_t* xsync = nullptr;  // [4]: arrivals by generation parity, generation
  uint32_t* rowmax = nullptr;  // [kDecodeMaxM][kRowMaxStride] row maxima of the decode kernel's own activation pass
  int32_t* idx = nullptr;
  int32_t* count = nullptr;
  float* colmax = nullptr;
  int* status = nullptr;
  // workspace sized by the largest M seen
  int64_t ws_rows = 0;
  int8_t* Xq = nullptr;
  float* c_x = nullptr;
  __half* X_OT = nullptr;
  // tensor map of Xq for the current (pointer, M, box rows)
  CUtensorMap tmA;
  const void* tmA_ptr = nullptr;
  int64_t tmA_rows = -1;
  int tmA_box = 0;
  // device copies for host-buffer forwards, and the stream and events that
  // copy Y out chunk by chunk while the next chunk computes
  int64_t io_rows = 0;
  __half* dX = nullptr;
  __half* dY = nullptr;
  cudaStream_t copy_stream = nullptr;
  cudaEvent_t chunk_ev[kHostChunks + 1] = {};
  // memory-saving weight (int8mm_prepare_weight_static): the stored fp16
  // rows, the row map, and per forward the gathered outlier rows, which the
  // GEMMs read as W with idx = 0, 1, 2, ...
  bool wstatic = false;
  int64_t w_rows = 0;
  int out_cap = 0;
  __half* Wc = nullptr;        // [w_rows][N]
  int32_t* wmap = nullptr;     // [K] slot in Wc, or -1
  int32_t* iota = nullptr;     // [out_cap] 0, 1, 2, ...
  __half* WO = nullptr;        // [out_cap][N]
  int32_t* count_w = nullptr;  // [1] min(|O|, out_cap)
  uint32_t* never_set = nullptr;  // [1] zero: the flag of the wait self-test
  unsigned long long timeout_ns = 2000000000ull;
  int test_skip = 0;  // INT8MM_TEST_SKIP_* bits (failure-detection tests only)
  size_t bytes = 0;
};

namespace {

thread_local std::string g_last_error;
std::mutex g_mu;
std::unordered_set<const int8mm_weight*> g_live;

int8mm_status fail(int8mm_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
int8mm_status fail(int8mm_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

int8mm_status cuda_fail(cudaError_t e, const char* what) {
  const int8mm_status s = (e == cudaErrorMemoryAllocation) ? INT8MM_ERR_OOM : INT8MM_ERR_CUDA;
  return fail(s, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool live(const int8mm_weight* h) {
  std::lock_guard<std::mutex> g(g_mu);
  return h != nullptr && g_live.count(h) != 0;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D int8 tensor [outer, inner] (inner contiguous), 128-byte swizzled boxes
// of box_inner x box_outer elements, zero fill outside the tensor.
int8mm_status make_tmap_i8(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                           uint32_t box_inner, uint32_t box_outer) {
  auto fn = encode_fn();
  if (fn == nullptr) return fail(INT8MM_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(INT8MM_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return INT8MM_OK;
}

template <typename T>
cudaError_t alloc(T** p, size_t count, cudaStream_t s, size_t* total) {
  *p = nullptr;
  if (count == 0) count = 1;
  cudaError_t e = cudaMallocAsync(reinterpret_cast<void**>(p), count * sizeof(T), s);
  if (e == cudaSuccess && total) *total += count * sizeof(T);
  return e;
}

template <typename T>
void release(T** p) {
  if (*p) cudaFree(*p);
  *p = nullptr;
}

void free_workspace(int8mm_weight* h) {
  release(&h->Xq);
  release(&h->c_x);
  release(&h->X_OT);
  h->ws_rows = 0;
  h->tmA_ptr = nullptr;
  h->tmA_rows = -1;
}

void free_all(int8mm_weight* h) {
  free_workspace(h);
  release(&h->dX);
  release(&h->dY);
  for (cudaEvent_t& ev : h->chunk_ev)
    if (ev) {
      cudaEventDestroy(ev);
      ev = nullptr;
    }
  if (h->copy_stream) {
    cudaStreamDestroy(h->copy_stream);
    h->copy_stream = nullptr;
  }
  release(&h->part);
  release(&h->dticket);
  release(&h->sk_ws);
  release(&h->sk_ticket);
  release(&h->Wb);
  release(&h->c_w);
  release(&h->inv_cw);
  release(&h->colmax_bits);
  release(&h->colkey);
  release(&h->epoch);
  release(&h->ticket);
  release(&h->mask);
  release(&h->pre);
  release(&h->omask);
  release(&h->xsync);
  release(&h->rowmax);
  release(&h->idx);
  release(&h->count);
  release(&h->colmax);
  release(&h->status);
  release(&h->Wc);
  release(&h->wmap);
  release(&h->iota);
  release(&h->WO);
  release(&h->count_w);
  release(&h->never_set);
}

// Row stride of X_OT for M rows: a multiple of 8, so that the GEMM reads
// 8 rows of an outlier column with one 16-byte load.
int64_t xot_stride(int64_t M) { return (M + 7) / 8 * 8; }

size_t ws_bytes(const int8mm_weight* h, int64_t rows) {
  return static_cast<size_t>(rows) * h->K                       // Xq
         + static_cast<size_t>(rows) * 4                        // c_x
         + static_cast<size_t>(xot_stride(rows)) * h->K * 2;    // X_OT
}

int8mm_status ensure_workspace(int8mm_weight* h, int64_t M, cudaStream_t s) {
  if (M <= h->ws_rows) return INT8MM_OK;
  int64_t rows = std::max<int64_t>(M, 2 * h->ws_rows);
  rows = std::max<int64_t>(rows, 128);
  // The old buffers may still be read by kernels enqueued earlier: free in
  // stream order on the same stream.
  if (h->ws_rows) {
    cudaFreeAsync(h->Xq, s);
    cudaFreeAsync(h->c_x, s);
    cudaFreeAsync(h->X_OT, s);
    h->bytes -= ws_bytes(h, h->ws_rows);
    h->Xq = nullptr;
    h->c_x = nullptr;
    h->X_OT = nullptr;
    h->ws_rows = 0;
  }
  cudaError_t e;
  if ((e = alloc(&h->Xq, static_cast<size_t>(rows) * h->K, s, nullptr)) != cudaSuccess ||
      (e = alloc(&h->c_x, static_cast<size_t>(rows), s, nullptr)) != cudaSuccess ||
      (e = alloc(&h->X_OT, static_cast<size_t>(xot_stride(rows)) * h->K, s, nullptr)) != cudaSuccess) {
    cudaStreamSynchronize(s);
    free_workspace(h);
    return cuda_fail(e, "workspace allocation");
  }
  h->ws_rows = rows;
  h->bytes += ws_bytes(h, rows);
  h->tmA_ptr = nullptr;
  h->tmA_rows = -1;
  return INT8MM_OK;
}

// Scratch of the decode GEMM (M <= kDecodeMaxM): int32 partial sums and
// per-n-block tickets, zeroed; allocated once, in stream order.
int8mm_status ensure_decode_scratch(int8mm_weight* h, cudaStream_t s) {
  if (h->part != nullptr) return INT8MM_OK;
  const size_t nb = static_cast<size_t>((h->N + 127) / 128);
  cudaError_t ea;
  if ((ea = alloc(&h->part, static_cast<size_t>(kDecodeMaxM) * h->N, s, &h->bytes)) != cudaSuccess ||
      (ea = alloc(&h->dticket, nb, s, &h->bytes)) != cudaSuccess ||
      (ea = cudaMemsetAsync(h->part, 0, static_cast<size_t>(kDecodeMaxM) * h->N * 4, s)) != cudaSuccess ||
      (ea = cudaMemsetAsync(h->dticket, 0, nb * 4, s)) != cudaSuccess) {
    cudaStreamSynchronize(s);
    release(&h->part);
    release(&h->dticket);
    return cuda_fail(ea, "decode scratch allocation");
  }
  return INT8MM_OK;
}

// Split K of the prefill GEMM for M rows (the handle's forced split, or
// the library's choice), and the scratch it needs: (pieces - 1) partial
// tiles per split tile and 4 tickets per split tile.
GemmSplit split_for(const int8mm_weight* h, int64_t M) {
  return gemm_split_for(M, h->N, h->K, h->num_sms, h->split_override);
}
size_t split_ws_elems(const GemmSplit& sp) {
  return sp.pieces > 1 ? static_cast<size_t>(sp.pieces - 1) * sp.tail * 2 * kGemmBM * kGemmBN : 0;
}
size_t split_tickets(const GemmSplit& sp) { return sp.pieces > 1 ? static_cast<size_t>(sp.tail) * 4 : 0; }

// Grows the split-K partial-tile workspace to ws_elems int32 and the tickets
// to n_tickets zeroed counters, in stream order (old buffers freed on s).
int8mm_status ensure_split_scratch(int8mm_weight* h, size_t ws_elems, size_t n_tickets, cudaStream_t s) {
  cudaError_t e;
  if (ws_elems > h->sk_ws_elems) {
    if (h->sk_ws) {
      cudaFreeAsync(h->sk_ws, s);
      h->bytes -= h->sk_ws_elems * 4;
      h->sk_ws = nullptr;
      h->sk_ws_elems = 0;
    }
    if ((e = alloc(&h->sk_ws, ws_elems, s, &h->bytes)) != cudaSuccess) {
      cudaStreamSynchronize(s);
      release(&h->sk_ws);
      return cuda_fail(e, "split-K workspace allocation");
    }
    h->sk_ws_elems = ws_elems;
  }
  if (n_tickets > h->sk_ticket_n) {
    if (h->sk_ticket) {
      cudaFreeAsync(h->sk_ticket, s);
      h->bytes -= h->sk_ticket_n * 4;
      h->sk_ticket = nullptr;
      h->sk_ticket_n = 0;
    }
    if ((e = alloc(&h->sk_ticket, n_tickets, s, &h->bytes)) != cudaSuccess ||
        (e = cudaMemsetAsync(h->sk_ticket, 0, n_tickets * 4, s)) != cudaSuccess) {
      cudaStreamSynchronize(s);
      release(&h->sk_ticket);
      return cuda_fail(e, "split-K ticket allocation");
    }
    h->sk_ticket_n = n_tickets;
  }
  return INT8MM_OK;
}

int8mm_status check_forward_args(const int8mm_weight* h, const void* X, int64_t M, float alpha, const void* Y) {
  if (!live(h)) return fail(INT8MM_ERR_INVALID_ARG, "invalid or freed weight handle");
  if (M < 0 || M >= (int64_t(1) << 31)) return fail(INT8MM_ERR_INVALID_ARG, "M=%lld out of range", (long long)M);
  if (std::isnan(alpha)) return fail(INT8MM_ERR_INVALID_ARG, "alpha is NaN");
  if (M == 0) return INT8MM_OK;
  if (X == nullptr || Y == nullptr) return fail(INT8MM_ERR_INVALID_ARG, "X or Y is NULL");
  const int64_t tiles = ((M + kGemmBM - 1) / kGemmBM) * ((h->N + kGemmBN - 1) / kGemmBN);
  const int64_t detect_blocks = ((h->K + 255) / 256) * ((M + 63) / 64);
  if (tiles >= (int64_t(1) << 31) || detect_blocks >= (int64_t(1) << 31) || M * h->N >= (int64_t(1) << 62))
    return fail(INT8MM_ERR_UNSUPPORTED_SHAPE, "M=%lld x N=%lld is too large", (long long)M, (long long)h->N);
  if (!aligned16(X) || !aligned16(Y)) return fail(INT8MM_ERR_ALIGNMENT, "X and Y must be 16-byte aligned");
  return INT8MM_OK;
}

int8mm_status set_device(const int8mm_weight* h) {
  int cur = -1;
  cudaGetDevice(&cur);
  if (cur != h->device) {
    cudaError_t e = cudaSetDevice(h->device);
    if (e != cudaSuccess) return cuda_fail(e, "cudaSetDevice");
  }
  return INT8MM_OK;
}

// With chunk_rows > 0, the prefill GEMM runs on row chunks of that many
// rows (a multiple of 256) and after_chunk(r0, rows) is called once each
// chunk's GEMM is enqueued; *whole tells the caller whether that happened
// (false for the decode GEMM, which runs once).
int8mm_status forward_impl(int8mm_weight* h, const void* X, int64_t M, float alpha, void* Y, cudaStream_t s,
                           void* const* events, const int8mm_debug_bufs* dbg, const void* bias = nullptr,
                           int64_t chunk_rows = 0,
                           const std::function<int8mm_status(int64_t, int64_t)>& after_chunk = nullptr,
                           bool* chunked = nullptr) {
  bool whole_done = false;
  int8mm_status st = check_forward_args(h, X, M, alpha, Y);
  if (st != INT8MM_OK) return st;
  if (M == 0) return INT8MM_OK;
  if ((st = set_device(h)) != INT8MM_OK) return st;
  if ((st = ensure_workspace(h, M, s)) != INT8MM_OK) return st;
  const bool decode = M <= kDecodeMaxM;
  const int64_t ld_xo = xot_stride(M);
  const int box_rows = decode ? decode_padded_tokens(M) : kGemmBM;
  if (h->tmA_ptr != h->Xq || h->tmA_rows != M || h->tmA_box != box_rows) {
    if ((st = make_tmap_i8(&h->tmA, h->Xq, h->K, M, kGemmBK, box_rows)) != INT8MM_OK) return st;
    h->tmA_ptr = h->Xq;
    h->tmA_rows = M;
    h->tmA_box = box_rows;
  }
  if (decode && (st = ensure_decode_scratch(h, s)) != INT8MM_OK) return st;
  OutlierScratch sc{h->colkey, h->epoch, h->ticket, h->mask, h->pre, h->idx, h->count, h->colmax};
  const __half* Xh = static_cast<const __half*>(X);
  cudaError_t e;
  auto rec = [&](int i) {
    if (events && events[i]) cudaEventRecord(static_cast<cudaEvent_t>(events[i]), s);
  };
  rec(0);
  // Decode shapes run the activation pass inside the decode GEMM's launch
  // (not with a static weight, whose outlier rows are gathered in between,
  // nor when events should time the two passes apart).
  const bool fused = decode && !h->wstatic && !(events && events[1]) &&
                     decode_fused_fits(M, h->K, h->N, h->num_sms);
  if (fused) {
    // the debug dump's column maxima come from the detection kernel
    if (dbg && (e = launch_outlier_detect(Xh, M, h->K, alpha, sc, s)) != cudaSuccess)
      return cuda_fail(e, "outlier detection launch");
  } else if (row_act_fits(M, h->K, h->num_sms)) {
    RowActArgs ra;
    ra.X = Xh;
    ra.M = static_cast<int>(M);
    ra.K = static_cast<int>(h->K);
    ra.rows_per_block = 0;
    ra.groups = 0;
    ra.thr = half_magnitude_threshold(alpha);
    ra.Xq = h->Xq;
    ra.c_x = h->c_x;
    ra.X_OT = h->X_OT;
    ra.ld_xo = static_cast<int>(ld_xo);
    ra.idx = h->idx;
    ra.count = h->count;
    ra.omask = h->omask;
    ra.sync = h->xsync;
    ra.status = h->status;
    ra.timeout_ns = h->timeout_ns;
    ra.skip_arrival = (h->test_skip & INT8MM_TEST_SKIP_BARRIER_ARRIVAL) != 0;
    // the debug dump's column maxima come from the detection kernel
    if (dbg && (e = launch_outlier_detect(Xh, M, h->K, alpha, sc, s)) != cudaSuccess)
      return cuda_fail(e, "outlier detection launch");
    if ((e = launch_row_act(ra, h->num_sms, s)) != cudaSuccess) return cuda_fail(e, "activation pass launch");
  } else {
    if ((e = launch_outlier_detect(Xh, M, h->K, alpha, sc, s)) != cudaSuccess)
      return cuda_fail(e, "outlier detection launch");
    if ((e = launch_row_quant(Xh, M, h->K, sc, h->Xq, h->c_x, h->X_OT, ld_xo, /*pdl=*/true, s)) != cudaSuccess)
      return cuda_fail(e, "row quantisation launch");
  }
  if (h->wstatic) {
    // this forward's outlier weight rows, in the order of idx
    GatherArgs ga{h->idx, h->count, h->wmap, h->Wc, h->Wb, h->inv_cw, static_cast<int>(h->N),
                  static_cast<int>(h->N_pad), h->out_cap, h->WO, h->count_w, h->status};
    if ((e = launch_gather_outlier_rows(ga, h->num_sms, /*pdl=*/true, s)) != cudaSuccess)
      return cuda_fail(e, "outlier row gather launch");
  }
  rec(1);
  // Without events between them, the GEMM is a programmatic dependent of the
  // row pass; an event record in between makes it an ordinary launch.
  const bool pdl = !(events && events[1]);
  // the GEMMs read the outlier product's weight rows as W[idx[o]]: the
  // borrowed W and the outlier columns, or the gathered rows and 0, 1, 2, ...
  const __half* Wrows = h->wstatic ? h->WO : h->W;
  const int32_t* widx = h->wstatic ? h->iota : h->idx;
  const int32_t* wcount = h->wstatic ? h->count_w : h->count;
  if (decode) {
    DecodeArgs d;
    d.M = static_cast<int>(M);
    d.N = static_cast<int>(h->N);
    d.K = static_cast<int>(h->K);
    d.N_pad = static_cast<int>(h->N_pad);
    d.c_x = h->c_x;
    d.inv_cw = h->inv_cw;
    d.W = Wrows;
    d.X_OT = h->X_OT;
    d.ld_xo = static_cast<int>(ld_xo);
    d.idx = widx;
    d.count = wcount;
    d.Y = static_cast<__half*>(Y);
    d.bias = static_cast<const __half*>(bias);
    d.acc_dump = dbg ? dbg->acc : nullptr;
    d.part = h->part;
    d.ticket = h->dticket;
    d.status = h->status;
    d.timeout_ns = h->timeout_ns;
    d.skip_arrival = (h->test_skip & INT8MM_TEST_SKIP_DECODE_TICKET) != 0;
    d.X = fused ? Xh : nullptr;
    d.thr = half_magnitude_threshold(alpha);
    d.Xq_out = h->Xq;
    d.c_x_out = h->c_x;
    d.X_OT_out = h->X_OT;
    d.idx_out = h->idx;
    d.count_out = h->count;
    d.omask = h->omask;
    d.sync = h->xsync;
    d.rowmax = h->rowmax;
    d.skip_barrier = (h->test_skip & INT8MM_TEST_SKIP_BARRIER_ARRIVAL) != 0;
    if ((e = launch_gemm_decode(h->tmW128, h->tmA, d, h->num_sms, pdl, s)) != cudaSuccess)
      return cuda_fail(e, "int8 decode GEMM launch");
  } else {
    // Rows [r0, r0 + rows) at a time (all of them unless the host-buffer
    // forward asks for chunks, to copy each chunk of Y out while the next
    // one computes); the first launch is the activation pass's dependent.
    const int64_t step = (chunk_rows > 0 && chunk_rows < M) ? chunk_rows : M;
    for (int64_t r0 = 0; r0 < M; r0 += step) {
      const int64_t rows = std::min(step, M - r0);
      // split K for the CTA-pair tiles; the scratch grows on demand
      const GemmSplit sp = split_for(h, rows);
      if (sp.pieces > 1 && (st = ensure_split_scratch(h, split_ws_elems(sp), split_tickets(sp), s)) != INT8MM_OK)
        return st;
      GemmArgs a;
      a.M = static_cast<int>(rows);
      a.a_row0 = static_cast<int>(r0);
      a.N = static_cast<int>(h->N);
      a.K = static_cast<int>(h->K);
      a.N_pad = static_cast<int>(h->N_pad);
      a.c_x = h->c_x + r0;
      a.inv_cw = h->inv_cw;
      a.W = Wrows;
      a.X_OT = h->X_OT + r0;
      a.ld_xo = static_cast<int>(ld_xo);
      a.idx = widx;
      a.count = wcount;
      a.Y = static_cast<__half*>(Y) + r0 * h->N;
      a.bias = static_cast<const __half*>(bias);
      a.acc_dump = dbg ? dbg->acc + r0 * h->N : nullptr;
      a.split = sp.pieces;
      a.tail_tiles = sp.pieces > 1 ? sp.tail : 0;
      a.sk_ws = h->sk_ws;
      a.sk_ticket = h->sk_ticket;
      a.status = h->status;
      a.timeout_ns = h->timeout_ns;
      a.skip_arrival = (h->test_skip & INT8MM_TEST_SKIP_SPLITK_TICKET) != 0;
      if ((e = launch_gemm_decomp(h->tmA, h->tmW128, a, h->num_sms, pdl && r0 == 0, s)) != cudaSuccess)
        return cuda_fail(e, "int8 GEMM launch");
      if (after_chunk && (st = after_chunk(r0, rows)) != INT8MM_OK) return st;
    }
    whole_done = true;
  }
  rec(2);
  if (chunked) *chunked = whole_done;
  if (dbg) {
    const size_t K = static_cast<size_t>(h->K), N = static_cast<size_t>(h->N), Mz = static_cast<size_t>(M);
    struct C {
      void* dst;
      const void* src;
      size_t n;
    } cps[] = {
        {dbg->colmax, h->colmax, K * 4},  {dbg->outlier_idx, h->idx, K * 4}, {dbg->outlier_count, h->count, 4},
        {dbg->x_codes, h->Xq, Mz * K},    {dbg->c_x, h->c_x, Mz * 4},
        {dbg->c_w, h->c_w, N * 4},
    };
    for (const C& c : cps)
      if (c.dst && (e = cudaMemcpyAsync(c.dst, c.src, c.n, cudaMemcpyDeviceToDevice, s)) != cudaSuccess)
        return cuda_fail(e, "debug copy");
    if (dbg->w_codes_t) {  // K-blocked [K/128][N_pad][128] -> [N, K]
      for (size_t kb = 0; kb * 128 < K; ++kb) {
        const size_t width = std::min<size_t>(128, K - kb * 128);
        if ((e = cudaMemcpy2DAsync(static_cast<int8_t*>(dbg->w_codes_t) + kb * 128, K,
                                   h->Wb + kb * static_cast<size_t>(h->N_pad) * 128, 128, width, N,
                                   cudaMemcpyDeviceToDevice, s)) != cudaSuccess)
          return cuda_fail(e, "debug copy of the weight codes");
      }
    }
  }
  return INT8MM_OK;
}

}  // namespace

void i8mm::set_last_error(const std::string& message) { g_last_error = message; }

namespace {

// Shared by both prepare entry points; with `wstatic`, the memory-saving
// weight keeping W[rows[i], :] for i < n_rows (validated by the caller).
int8mm_status prepare_impl(const void* W_fp16_dev, int64_t K, int64_t N, void* stream, int8mm_weight_t* out,
                           bool wstatic, const int32_t* rows, int64_t n_rows, int max_outliers) {
  if (out == nullptr) return fail(INT8MM_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (W_fp16_dev == nullptr) return fail(INT8MM_ERR_INVALID_ARG, "W is NULL");
  if (K < 16 || N < 16 || K % 16 != 0 || N % 16 != 0 || K > INT8MM_MAX_K || N >= (int64_t(1) << 31))
    return fail(INT8MM_ERR_UNSUPPORTED_SHAPE,
                "K=%lld, N=%lld: need 16 <= K <= %d and N >= 16, both multiples of 16", (long long)K,
                (long long)N, INT8MM_MAX_K);
  if (!aligned16(W_fp16_dev)) return fail(INT8MM_ERR_ALIGNMENT, "W must be 16-byte aligned");
  if ((K + 127) / 128 * ((N + kWeightRowPad - 1) / kWeightRowPad * kWeightRowPad) >= (int64_t(1) << 31))
    return fail(INT8MM_ERR_UNSUPPORTED_SHAPE, "K=%lld x N=%lld exceeds the weight layout's 2^31 rows of 128 bytes",
                (long long)K, (long long)N);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int8mm_weight* h = new int8mm_weight();
  cudaError_t e = cudaGetDevice(&h->device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device);
  if (e != cudaSuccess) {
    delete h;
    return cuda_fail(e, "device query");
  }
  h->K = K;
  h->N = N;
  h->W = static_cast<const __half*>(W_fp16_dev);
  const size_t Kz = static_cast<size_t>(K), Nz = static_cast<size_t>(N);
  const size_t words = (Kz + 31) / 32;
  size_t* tot = &h->bytes;
  h->N_pad = (N + kWeightRowPad - 1) / kWeightRowPad * kWeightRowPad;
  const size_t kblocks = (Kz + 127) / 128;
  const size_t wb_bytes = kblocks * static_cast<size_t>(h->N_pad) * 128;
  if ((e = alloc(&h->Wb, wb_bytes, s, tot)) != cudaSuccess || (e = alloc(&h->c_w, Nz, s, tot)) != cudaSuccess ||
      (e = alloc(&h->inv_cw, Nz, s, tot)) != cudaSuccess || (e = alloc(&h->colmax_bits, Nz, s, tot)) != cudaSuccess ||
      (e = alloc(&h->colkey, Kz, s, tot)) != cudaSuccess || (e = alloc(&h->epoch, 1, s, tot)) != cudaSuccess ||
      (e = alloc(&h->ticket, 1, s, tot)) != cudaSuccess || (e = alloc(&h->mask, words, s, tot)) != cudaSuccess ||
      (e = alloc(&h->pre, words, s, tot)) != cudaSuccess || (e = alloc(&h->omask, 2 * words, s, tot)) != cudaSuccess ||
      (e = alloc(&h->xsync, 4, s, tot)) != cudaSuccess || (e = alloc(&h->rowmax, kDecodeMaxM * kRowMaxStride, s, tot)) != cudaSuccess ||
      (e = alloc(&h->idx, Kz, s, tot)) != cudaSuccess ||
      (e = alloc(&h->count, 1, s, tot)) != cudaSuccess || (e = alloc(&h->colmax, Kz, s, tot)) != cudaSuccess ||
      (e = alloc(&h->status, 1, s, tot)) != cudaSuccess) {
    cudaStreamSynchronize(s);
    free_all(h);
    delete h;
    return cuda_fail(e, "weight allocation");
  }
  if ((e = cudaMemsetAsync(h->Wb, 0, wb_bytes, s)) != cudaSuccess ||
      (e = cudaMemsetAsync(h->colkey, 0, Kz * 8, s)) != cudaSuccess ||
      (e = cudaMemsetAsync(h->epoch, 0, 8, s)) != cudaSuccess ||
      (e = cudaMemsetAsync(h->ticket, 0, 4, s)) != cudaSuccess ||
      (e = cudaMemsetAsync(h->mask, 0, words * 4, s)) != cudaSuccess ||
      (e = cudaMemsetAsync(h->omask, 0, 2 * words * 4, s)) != cudaSuccess ||
      (e = cudaMemsetAsync(h->xsync, 0, 16, s)) != cudaSuccess ||
      (e = cudaMemsetAsync(h->rowmax, 0, kDecodeMaxM * kRowMaxStride * 4, s)) != cudaSuccess ||
      (e = cudaMemsetAsync(h->count, 0, 4, s)) != cudaSuccess ||
      (e = cudaMemsetAsync(h->status, 0, 4, s)) != cudaSuccess ||
      (e = launch_weight_prep(h->W, K, N, h->colmax_bits, h->Wb, h->N_pad, h->c_w, h->inv_cw, h->num_sms, s)) !=
          cudaSuccess) {
    cudaStreamSynchronize(s);
    free_all(h);
    delete h;
    return cuda_fail(e, "weight preparation");
  }
  const uint64_t wb_rows = kblocks * static_cast<uint64_t>(h->N_pad);
  int8mm_status st = make_tmap_i8(&h->tmW128, h->Wb, 128, wb_rows, kGemmBK, 128);
  if (st == INT8MM_OK && wstatic) {
    // the stored rows and the row map; W is not kept
    std::vector<int32_t> wmap(Kz, -1), iota(static_cast<size_t>(max_outliers));
    for (int64_t i = 0; i < n_rows; ++i) wmap[static_cast<size_t>(rows[i])] = static_cast<int32_t>(i);
    for (int i = 0; i < max_outliers; ++i) iota[static_cast<size_t>(i)] = i;
    const size_t R = static_cast<size_t>(n_rows), cap = static_cast<size_t>(max_outliers);
    h->wstatic = true;
    h->w_rows = n_rows;
    h->out_cap = max_outliers;
    if ((e = alloc(&h->Wc, R * Nz, s, tot)) != cudaSuccess || (e = alloc(&h->wmap, Kz, s, tot)) != cudaSuccess ||
        (e = alloc(&h->iota, cap, s, tot)) != cudaSuccess || (e = alloc(&h->WO, cap * Nz, s, tot)) != cudaSuccess ||
        (e = alloc(&h->count_w, 1, s, tot)) != cudaSuccess) {
      st = cuda_fail(e, "static weight allocation");
    } else {
      for (size_t i = 0; i < R && e == cudaSuccess; ++i)
        e = cudaMemcpyAsync(h->Wc + i * Nz, h->W + static_cast<size_t>(rows[i]) * Nz, Nz * 2,
                            cudaMemcpyDeviceToDevice, s);
      if (e == cudaSuccess) e = cudaMemcpyAsync(h->wmap, wmap.data(), Kz * 4, cudaMemcpyHostToDevice, s);
      if (e == cudaSuccess) e = cudaMemcpyAsync(h->iota, iota.data(), cap * 4, cudaMemcpyHostToDevice, s);
      // the host vectors and the caller's W must outlive the copies
      if (e == cudaSuccess) e = cudaStreamSynchronize(s);
      if (e != cudaSuccess) st = cuda_fail(e, "static weight rows");
    }
    h->W = nullptr;
  }
  if (st != INT8MM_OK) {
    cudaStreamSynchronize(s);
    free_all(h);
    delete h;
    return st;
  }
  {
    std::lock_guard<std::mutex> g(g_mu);
    g_live.insert(h);
  }
  *out = h;
  return INT8MM_OK;
}

}  // namespace

extern "C" {

int8mm_status int8mm_prepare_weight(const void* W_fp16_dev, int64_t K, int64_t N, void* stream,
                                    int8mm_weight_t* out) {
  return prepare_impl(W_fp16_dev, K, N, stream, out, false, nullptr, 0, 0);
}

int8mm_status int8mm_prepare_weight_static(const void* W_fp16_dev, int64_t K, int64_t N, const int32_t* rows,
                                           int64_t n_rows, int max_outliers, void* stream, int8mm_weight_t* out) {
  if (out == nullptr) return fail(INT8MM_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (K < 16 || K > INT8MM_MAX_K)  // the shape error, from the common checks
    return prepare_impl(W_fp16_dev, K, N, stream, out, true, rows, 0, 1);
  if (n_rows < 0 || n_rows > K || (n_rows > 0 && rows == nullptr))
    return fail(INT8MM_ERR_INVALID_ARG, "n_rows=%lld: need 0 <= n_rows <= K and rows given", (long long)n_rows);
  if (max_outliers < 1 || max_outliers > K)
    return fail(INT8MM_ERR_INVALID_ARG, "max_outliers=%d: need 1 <= max_outliers <= K", max_outliers);
  std::vector<char> seen(static_cast<size_t>(K), 0);
  for (int64_t i = 0; i < n_rows; ++i) {
    if (rows[i] < 0 || rows[i] >= K || seen[static_cast<size_t>(rows[i])])
      return fail(INT8MM_ERR_INVALID_ARG, "rows[%lld]=%d: need distinct input dimensions in [0, K)", (long long)i,
                  rows[i]);
    seen[static_cast<size_t>(rows[i])] = 1;
  }
  return prepare_impl(W_fp16_dev, K, N, stream, out, true, rows, n_rows, max_outliers);
}

int8mm_status int8mm_reserve(int8mm_weight_t h, int64_t M_max, void* stream) {
  if (!live(h)) return fail(INT8MM_ERR_INVALID_ARG, "invalid or freed weight handle");
  if (M_max < 0 || M_max >= (int64_t(1) << 31)) return fail(INT8MM_ERR_INVALID_ARG, "M_max out of range");
  int8mm_status st = set_device(h);
  if (st != INT8MM_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = ensure_workspace(h, M_max, s)) != INT8MM_OK) return st;
  if (M_max >= 1 && (st = ensure_decode_scratch(h, s)) != INT8MM_OK) return st;
  // the largest split-K scratch of any M <= M_max (the split depends on M
  // only through its number of 256-row tiles)
  size_t ws_max = 0, tickets_max = 0;
  for (int64_t mt = 1; (mt - 1) * 2 * kGemmBM < M_max; ++mt) {
    const int64_t M = std::min<int64_t>(M_max, mt * 2 * kGemmBM);
    if (M <= kDecodeMaxM) continue;  // the decode GEMM: no split
    const GemmSplit sp = split_for(h, M);
    ws_max = std::max(ws_max, split_ws_elems(sp));
    tickets_max = std::max(tickets_max, split_tickets(sp));
  }
  if (ws_max > 0) return ensure_split_scratch(h, ws_max, tickets_max, s);
  return INT8MM_OK;
}

int8mm_status int8mm_forward(int8mm_weight_t h, const void* X_fp16_dev, int64_t M, float alpha, void* Y_fp16_dev,
                             void* stream) {
  return forward_impl(h, X_fp16_dev, M, alpha, Y_fp16_dev, static_cast<cudaStream_t>(stream), nullptr, nullptr);
}

int8mm_status int8mm_forward_bias(int8mm_weight_t h, const void* X_fp16_dev, int64_t M, float alpha,
                                  const void* bias_fp16_dev, void* Y_fp16_dev, void* stream) {
  if (bias_fp16_dev != nullptr && !aligned16(bias_fp16_dev))
    return fail(INT8MM_ERR_ALIGNMENT, "bias must be 16-byte aligned");
  return forward_impl(h, X_fp16_dev, M, alpha, Y_fp16_dev, static_cast<cudaStream_t>(stream), nullptr, nullptr,
                      bias_fp16_dev);
}

int8mm_status int8mm_forward_events(int8mm_weight_t h, const void* X_fp16_dev, int64_t M, float alpha,
                                    void* Y_fp16_dev, void* stream, void* const events[3]) {
  return forward_impl(h, X_fp16_dev, M, alpha, Y_fp16_dev, static_cast<cudaStream_t>(stream), events, nullptr);
}

int8mm_status int8mm_forward_debug(int8mm_weight_t h, const void* X_fp16_dev, int64_t M, float alpha,
                                   void* Y_fp16_dev, void* stream, const int8mm_debug_bufs* dbg) {
  if (dbg && dbg->acc && !aligned16(dbg->acc)) return fail(INT8MM_ERR_ALIGNMENT, "dbg->acc must be 16-byte aligned");
  return forward_impl(h, X_fp16_dev, M, alpha, Y_fp16_dev, static_cast<cudaStream_t>(stream), nullptr, dbg);
}

int8mm_status int8mm_forward_host(int8mm_weight_t h, const void* X_fp16_host, int64_t M, float alpha,
                                  void* Y_fp16_host, void* stream) {
  int8mm_status st = check_forward_args(h, X_fp16_host, M, 0.0f, Y_fp16_host);
  if (st != INT8MM_OK) return st;
  if (std::isnan(alpha)) return fail(INT8MM_ERR_INVALID_ARG, "alpha is NaN");
  if (M == 0) return INT8MM_OK;
  if ((st = set_device(h)) != INT8MM_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (M > h->io_rows) {
    if (h->io_rows) {
      cudaFreeAsync(h->dX, s);
      cudaFreeAsync(h->dY, s);
      h->bytes -= static_cast<size_t>(h->io_rows) * (h->K + h->N) * 2;
      h->dX = h->dY = nullptr;
      h->io_rows = 0;
    }
    if ((e = alloc(&h->dX, static_cast<size_t>(M) * h->K, s, nullptr)) != cudaSuccess ||
        (e = alloc(&h->dY, static_cast<size_t>(M) * h->N, s, nullptr)) != cudaSuccess) {
      cudaStreamSynchronize(s);
      release(&h->dX);
      release(&h->dY);
      return cuda_fail(e, "host-forward buffers");
    }
    h->io_rows = M;
    h->bytes += static_cast<size_t>(M) * (h->K + h->N) * 2;
  }
  if ((e = cudaMemcpyAsync(h->dX, X_fp16_host, static_cast<size_t>(M) * h->K * 2, cudaMemcpyHostToDevice, s)) !=
      cudaSuccess)
    return cuda_fail(e, "copy of X to the device");
  const size_t row_bytes = static_cast<size_t>(h->N) * 2;
  // Tall prefills: the GEMM runs in kHostChunks row chunks (multiples of its
  // 256-row tiles) and each chunk of Y goes back on a second stream as soon
  // as it is written, overlapping the read-back with the next chunks (the
  // activation pass needs all of X, so the upload stays in front).
  const int64_t chunk = (M + kHostChunks - 1) / kHostChunks;
  const int64_t chunk_rows = (chunk + 2 * kGemmBM - 1) / (2 * kGemmBM) * (2 * kGemmBM);
  if (M > kDecodeMaxM && M >= 2 * chunk_rows) {
    if (h->copy_stream == nullptr) {
      if ((e = cudaStreamCreateWithFlags(&h->copy_stream, cudaStreamNonBlocking)) != cudaSuccess)
        return cuda_fail(e, "copy stream");
      for (cudaEvent_t& ev : h->chunk_ev)
        if ((e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming)) != cudaSuccess)
          return cuda_fail(e, "copy events");
    }
    int n = 0;
    auto copy_out = [&](int64_t r0, int64_t rows) -> int8mm_status {
      cudaError_t ce;
      if ((ce = cudaEventRecord(h->chunk_ev[n], s)) != cudaSuccess ||
          (ce = cudaStreamWaitEvent(h->copy_stream, h->chunk_ev[n], 0)) != cudaSuccess ||
          (ce = cudaMemcpyAsync(static_cast<char*>(Y_fp16_host) + static_cast<size_t>(r0) * row_bytes,
                                reinterpret_cast<char*>(h->dY) + static_cast<size_t>(r0) * row_bytes,
                                static_cast<size_t>(rows) * row_bytes, cudaMemcpyDeviceToHost, h->copy_stream)) !=
              cudaSuccess)
        return cuda_fail(ce, "copy of Y to the host");
      ++n;
      return INT8MM_OK;
    };
    bool chunked = false;
    if ((st = forward_impl(h, h->dX, M, alpha, h->dY, s, nullptr, nullptr, nullptr, chunk_rows, copy_out,
                           &chunked)) != INT8MM_OK)
      return st;
    if (chunked) {
      // `stream` is done once every chunk has arrived
      if ((e = cudaEventRecord(h->chunk_ev[kHostChunks], h->copy_stream)) != cudaSuccess ||
          (e = cudaStreamWaitEvent(s, h->chunk_ev[kHostChunks], 0)) != cudaSuccess)
        return cuda_fail(e, "copy of Y to the host");
      return INT8MM_OK;
    }
  } else if ((st = forward_impl(h, h->dX, M, alpha, h->dY, s, nullptr, nullptr)) != INT8MM_OK) {
    return st;
  }
  if ((e = cudaMemcpyAsync(Y_fp16_host, h->dY, static_cast<size_t>(M) * row_bytes, cudaMemcpyDeviceToHost, s)) !=
      cudaSuccess)
    return cuda_fail(e, "copy of Y to the host");
  return INT8MM_OK;
}

int8mm_status int8mm_get_status(int8mm_weight_t h) {
  if (!live(h)) return fail(INT8MM_ERR_INVALID_ARG, "invalid or freed weight handle");
  int8mm_status st = set_device(h);
  if (st != INT8MM_OK) return st;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "device synchronise");
  int word = 0;
  if ((e = cudaMemcpy(&word, h->status, 4, cudaMemcpyDeviceToHost)) != cudaSuccess)
    return cuda_fail(e, "status read");
  if ((e = cudaMemset(h->status, 0, 4)) != cudaSuccess) return cuda_fail(e, "status reset");
  if ((e = cudaDeviceSynchronize()) != cudaSuccess) return cuda_fail(e, "device synchronise");
  if (word & kStatusTimeout) {
    // an aborted decode GEMM may leave partial sums and tickets behind,
    if (h->part) cudaMemset(h->part, 0, static_cast<size_t>(kDecodeMaxM) * h->N * 4);
    if (h->dticket) cudaMemset(h->dticket, 0, static_cast<size_t>((h->N + 127) / 128) * 4);
    // an aborted split-K GEMM its tile tickets,
    if (h->sk_ticket) cudaMemset(h->sk_ticket, 0, h->sk_ticket_n * 4);
    // and an aborted single-launch activation pass (separate or inside the
    // decode GEMM) its barrier counts, bitmasks and row maxima
    cudaMemset(h->xsync, 0, 16);
    cudaMemset(h->rowmax, 0, kDecodeMaxM * kRowMaxStride * 4);
    cudaMemset(h->omask, 0, static_cast<size_t>((h->K + 31) / 32) * 8);
    cudaDeviceSynchronize();
    return fail(INT8MM_ERR_TIMEOUT, "a device wait ran out of time");
  }
  if (word & kStatusOutlierCap)
    return fail(INT8MM_ERR_OUTLIER_CAP, "a forward found more than the static weight's %d outlier columns",
                h->out_cap);
  return INT8MM_OK;
}

int8mm_status int8mm_set_wait_limit(int8mm_weight_t h, uint64_t timeout_ns) {
  if (!live(h)) return fail(INT8MM_ERR_INVALID_ARG, "invalid or freed weight handle");
  // a block that gives up still waits, within this limit, for the copies and
  // MMAs it has issued (microseconds); the floor keeps that drain complete
  if (timeout_ns < 1000000ull)
    return fail(INT8MM_ERR_INVALID_ARG, "timeout %llu ns is below the 1 ms minimum",
                static_cast<unsigned long long>(timeout_ns));
  h->timeout_ns = timeout_ns;
  return INT8MM_OK;
}

int8mm_status int8mm_wait_selftest(int8mm_weight_t h, void* stream) {
  if (!live(h)) return fail(INT8MM_ERR_INVALID_ARG, "invalid or freed weight handle");
  int8mm_status st = set_device(h);
  if (st != INT8MM_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (h->never_set == nullptr) {
    if ((e = alloc(&h->never_set, 1, s, &h->bytes)) != cudaSuccess ||
        (e = cudaMemsetAsync(h->never_set, 0, 4, s)) != cudaSuccess) {
      cudaStreamSynchronize(s);
      release(&h->never_set);
      return cuda_fail(e, "self-test flag allocation");
    }
  }
  if ((e = launch_wait_selftest(h->never_set, h->status, h->timeout_ns, s)) != cudaSuccess)
    return cuda_fail(e, "wait self-test launch");
  return INT8MM_OK;
}

int8mm_status int8mm_set_test_skip(int8mm_weight_t h, int bits) {
  if (!live(h)) return fail(INT8MM_ERR_INVALID_ARG, "invalid or freed weight handle");
  const int all = INT8MM_TEST_SKIP_SPLITK_TICKET | INT8MM_TEST_SKIP_DECODE_TICKET | INT8MM_TEST_SKIP_BARRIER_ARRIVAL;
  if ((bits & ~all) != 0) return fail(INT8MM_ERR_INVALID_ARG, "unknown test bits 0x%x", bits);
  h->test_skip = bits;
  return INT8MM_OK;
}

int8mm_status int8mm_set_split_k(int8mm_weight_t h, int split) {
  if (!live(h)) return fail(INT8MM_ERR_INVALID_ARG, "invalid or freed weight handle");
  if (split < 0 || split > kGemmMaxSplit) return fail(INT8MM_ERR_INVALID_ARG, "split %d outside 0..%d", split, kGemmMaxSplit);
  h->split_override = split;
  return INT8MM_OK;
}

int8mm_status int8mm_weight_bytes(int8mm_weight_t h, size_t* bytes) {
  if (!live(h) || bytes == nullptr) return fail(INT8MM_ERR_INVALID_ARG, "invalid handle or NULL output");
  *bytes = h->bytes;
  return INT8MM_OK;
}

int8mm_status int8mm_launches_per_forward(int8mm_weight_t h, int64_t M, int* count) {
  if (!live(h) || count == nullptr) return fail(INT8MM_ERR_INVALID_ARG, "invalid handle or NULL output");
  if (M < 0) return fail(INT8MM_ERR_INVALID_ARG, "M=%lld is negative", (long long)M);
  if (M == 0) *count = 0;
  else if (M <= kDecodeMaxM && !h->wstatic && decode_fused_fits(M, h->K, h->N, h->num_sms)) *count = 1;
  else *count = row_act_fits(M, h->K, h->num_sms) ? 2 : 3;
  if (M > 0 && h->wstatic) *count += 1;  // the outlier row gather
  return INT8MM_OK;
}

void int8mm_free(int8mm_weight_t h) {
  if (h == nullptr) return;
  {
    std::lock_guard<std::mutex> g(g_mu);
    if (g_live.erase(h) == 0) return;
  }
  int cur = -1;
  cudaGetDevice(&cur);
  cudaSetDevice(h->device);
  cudaDeviceSynchronize();
  free_all(h);
  if (cur >= 0) cudaSetDevice(cur);
  delete h;
}

const char* int8mm_last_error(void) { return g_last_error.c_str(); }

}  // extern "C"
