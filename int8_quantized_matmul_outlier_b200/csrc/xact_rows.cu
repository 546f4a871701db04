// Activation pass for many rows in one launch: outlier-column detection,
// vector-wise row quantisation and the fp16 outlier gather, for activations
// that fit in the shared memory of the GPU's SMs.
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
// SM); block b owns the R consecutive rows [b R, b R + R) and copies them into
// its shared memory with bulk copies, one mbarrier per row.  Each thread owns
// a fixed set of 8-column vectors (for all of its rows, or of one row group).
// Then:
//   1. per 8-column vector, the max |x| over the block's rows; a column with
//      an entry above alpha sets its bit in the block's bitmask, and the
//      non-zero words are OR-ed into a global bitmask.  Since every entry of a
//      column not in O is at most alpha, "some entry above alpha" is exactly
//      "column maximum above alpha".
//   2. grid barrier: each block adds 1 (release) to the arrival counter of the
//      current generation's parity and waits (acquire) until it reaches G.
//      Block 0 then zeroes the other parity's counter and advances the
//      generation; no block reads either again in this launch.
//   3. every block reads the global bitmask and forms the prefix of its word
//      popcounts (the slot of an outlier column); block 0 writes the
//      ascending index list and the count.  From shared memory: per row the
//      absmax over the non-outlier columns and c_x; then the codes and the
//      outlier entries.
// The global bitmask is double-buffered by the parity of the generation:
// block 0 clears the buffer of the next generation, so no launch needs a
// clearing pass and all state stays on the device.
#include "actq.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

#include <algorithm>
#include <cmath>

namespace i8mm {
namespace {

constexpr int kMaxThreads = 1024;

// Thread (g, t), g = tid / CT, t = tid % CT, owns the 8-column vectors
// v = t + i CT (i < VPT) of the rows j = g, g + RG, .. of its block (RG row
// groups of CT threads, CT a multiple of 32).  Everything a thread needs about
// its columns (outlier flags, code masks, outlier slots) is fixed for all rows.
template <int VPT>
__global__ void __launch_bounds__(kMaxThreads, 1) xact_rows_kernel(RowActArgs a) {
  extern __shared__ __align__(128) unsigned char sm[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int NT = blockDim.x;
  const int CT = a.col_threads, RG = NT / CT;
  const int g = tid / CT, t = tid - g * CT;
  const int K = a.K, M = a.M, R = a.rows_per_block, H = a.chunk_rows, S = a.slots;
  const int nvec = K / 8, KW = (K + 31) / 32;
  const int r0 = static_cast<int>(blockIdx.x) * R;
  const int nr = min(R, M - r0);
  const int nch = (nr + H - 1) / H;  // chunks of this block's rows
  const bool streaming = nch > 1;    // rows pass through the slots twice
  const uint32_t row_bytes = 2u * static_cast<uint32_t>(K);

  uint4* xs = reinterpret_cast<uint4*>(sm);                                           // [S][nvec]
  uint32_t* mask_s = reinterpret_cast<uint32_t*>(sm + static_cast<size_t>(S) * row_bytes);  // [KW]
  int* pre_s = reinterpret_cast<int*>(mask_s + KW);                                   // [KW]
  uint32_t* rowmax_s = reinterpret_cast<uint32_t*>(pre_s + KW);                       // [H]
  float* c_s = reinterpret_cast<float*>(rowmax_s + H);                                // [H]
  uint64_t* bars = reinterpret_cast<uint64_t*>(rowmax_s + ((2 * H + 1) & ~1));          // [S], 8-byte aligned
  __shared__ uint32_t s_gen;
  __shared__ unsigned long long s_epoch;
  __shared__ int s_ok;

  // Chunk c (rows c H .. c H + H - 1 of the block) lives in half c % 2 of the
  // slots when streaming, else in slots 0 .. nr - 1.  The mbarrier of a slot
  // completes one phase per copy into it.  Only the last chunk can be short,
  // so in pass 1 row i of chunk c is copy c / 2 into its slot, and in pass 2
  // it follows the pass-1 copies into that slot (one fewer for the slots the
  // short last chunk leaves out).
  const int rc_last = nr - (nch - 1) * H;
  auto slot_of = [&](int c, int i) { return streaming ? (c & 1) * H + i : i; };
  auto parity = [&](int pass, int c, int i) -> uint32_t {
    if (!streaming) return 0u;
    if (pass == 1) return static_cast<uint32_t>((c >> 1) & 1);
    const int h = c & 1;
    const int n1 = (nch - h + 1) / 2 - ((((nch - 1) & 1) == h && i >= rc_last) ? 1 : 0);
    return static_cast<uint32_t>((n1 + (c >> 1)) & 1);
  };
  int last_c[2] = {-1, -1}, last_pass[2] = {0, 0};  // thread 0: the latest copy into each half
  auto issue = [&](int pass, int c) {  // thread 0: bulk copies of chunk c's rows
    last_c[c & 1] = c;
    last_pass[c & 1] = pass;
    const int rb = c * H, rc = min(H, nr - rb);
    const unsigned char* src =
        reinterpret_cast<const unsigned char*>(a.X) + static_cast<size_t>(r0 + rb) * row_bytes;
    for (int i = 0; i < rc; ++i) {
      uint64_t* b = &bars[slot_of(c, i)];
      mbar_arrive_expect_tx(b, row_bytes);
      bulk_load_1d(xs + static_cast<size_t>(slot_of(c, i)) * nvec, src + static_cast<size_t>(i) * row_bytes,
                   row_bytes, b);
    }
  };
  // waits (bounded) for chunk c's rows of the given pass; any thread
  auto wait_chunk = [&](int pass, int c) -> bool {
    const int rc = min(H, nr - c * H);
    for (int i = 0; i < rc; ++i)
      if (!mbar_wait(&bars[slot_of(c, i)], parity(pass, c, i), a.timeout_ns, nullptr)) return false;
    return true;
  };
  // thread 0, after a failed wait: let the copies still in flight land
  auto drain = [&]() {
    for (int h = 0; h < 2; ++h)
      if (last_c[h] >= 0) wait_chunk(last_pass[h], last_c[h]);
  };

  // The GEMM that follows may launch now; its blocks take the SMs this
  // kernel leaves.
  pdl_launch_dependents();
  if (tid == 0) {
    s_gen = *reinterpret_cast<volatile uint32_t*>(a.sync + 2);
    s_epoch = *reinterpret_cast<volatile unsigned long long*>(a.epoch);
    for (int j = 0; j < S; ++j) mbar_init(&bars[j], 1);
    fence_mbar_init();
  }
  for (int w = tid; w < KW; w += NT) mask_s[w] = 0u;
  for (int j = tid; j < H; j += NT) rowmax_s[j] = 0u;
  __syncthreads();
  if (tid == 0) {
    issue(1, 0);
    if (streaming) issue(1, 1);
  }

  // ------------------------------------------------------------- phase 1
  // max |x| of the owned vectors over the group's rows, as rows land; a
  // streamed half is refilled once every thread is done with it
  uint32_t mx[VPT][4];
#pragma unroll
  for (int i = 0; i < VPT; ++i) mx[i][0] = mx[i][1] = mx[i][2] = mx[i][3] = 0u;
  int ok = 1;
  for (int c = 0; c < nch; ++c) {
    const int rc = min(H, nr - c * H);
    for (int i = g; i < rc && ok; i += RG) {
      const int sl = slot_of(c, i);
      if (!mbar_wait(&bars[sl], parity(1, c, i), a.timeout_ns, nullptr)) {
        ok = 0;
        break;
      }
      const uint4* row = xs + static_cast<size_t>(sl) * nvec;
#pragma unroll
      for (int i2 = 0; i2 < VPT; ++i2) {
        const int v = t + i2 * CT;
        if (v < nvec) {
          const uint4 x = row[v];
          mx[i2][0] = __vmaxu2(mx[i2][0], x.x & 0x7fff7fffu);
          mx[i2][1] = __vmaxu2(mx[i2][1], x.y & 0x7fff7fffu);
          mx[i2][2] = __vmaxu2(mx[i2][2], x.z & 0x7fff7fffu);
          mx[i2][3] = __vmaxu2(mx[i2][3], x.w & 0x7fff7fffu);
        }
      }
    }
    if (streaming) {
      ok = __syncthreads_and(ok);  // the half is free
      if (tid == 0 && ok && c + 2 < nch) issue(1, c + 2);
    }
  }
  // a column is an outlier when some entry exceeds alpha; row groups OR
  // their flags into the block's bitmask
  const bool all_out = a.thr < 0;  // alpha < 0: every column is an outlier
  const uint32_t thr2 = all_out ? 0u : (static_cast<uint32_t>(a.thr) * 0x00010001u);
  const unsigned long long tag = s_epoch << 16;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int v = t + i * CT;
    if (v < nvec && ok) {
      uint32_t fl = 0;
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const uint32_t gt = all_out ? 0xffffffffu : __vcmpgtu2(mx[i][p], thr2);
        fl |= ((gt & 1u) << (2 * p)) | (((gt >> 16) & 1u) << (2 * p + 1));
      }
      if (fl) atomicOr(&mask_s[v >> 2], fl << ((v & 3) * 8));
      if (a.colkey != nullptr) {  // column maxima for the debug dump
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          atomicMax(a.colkey + 8 * v + 2 * p, tag | (mx[i][p] & 0xffffu));
          atomicMax(a.colkey + 8 * v + 2 * p + 1, tag | (mx[i][p] >> 16));
        }
      }
    }
  }
  ok = __syncthreads_and(ok);
  // streaming: the second pass's first two chunks load during the barrier
  if (streaming && tid == 0 && ok) {
    issue(2, 0);
    issue(2, 1);
  }
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
  if (!s_ok) {
    // leave no bulk copy in flight into this block's shared memory
    if (tid == 0) drain();
    return;
  }
  if (blockIdx.x == 0 && tid == 0) {
    // every block has read the generation and the epoch (before arriving)
    a.sync[(gen + 1u) & 1u] = 0u;
    a.sync[2] = gen + 1u;
    *a.epoch = s_epoch + 1;
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
      if (blockIdx.x == 0) {
        uint32_t bits = mask_s[w];
        int o = pos;
        while (bits) {
          a.idx[o++] = w * 32 + __ffs(bits) - 1;
          bits &= bits - 1;
        }
      }
      pos += __popc(mask_s[w]);
    }
    if (blockIdx.x == 0 && lane == 31) *a.count = incl;
  }
  if (blockIdx.x == 0) {
    uint32_t* next = a.omask + static_cast<size_t>((gen + 1u) & 1u) * KW;
    for (int w = tid; w < KW; w += NT) next[w] = 0u;
    if (a.colkey != nullptr)
      for (int c = tid; c < K; c += NT) {
        const unsigned long long key = __ldcg(a.colkey + c);
        a.colmax[c] = (key >> 16) == s_epoch
                          ? __half2float(__ushort_as_half(static_cast<unsigned short>(key & 0xffffu)))
                          : 0.0f;
      }
  }
  __syncthreads();
  // per owned vector: outlier flags, the masks that keep its non-outlier codes,
  // and the X_OT slot of its first outlier column
  uint32_t fl[VPT], keep[VPT][2];
  int slot[VPT];
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int v = t + i * CT;
    fl[i] = 0u;
    keep[i][0] = keep[i][1] = 0u;
    slot[i] = 0;
    if (v < nvec) {
      const int w = v >> 2, sh = (v & 3) * 8;
      fl[i] = (mask_s[w] >> sh) & 0xffu;
      keep[i][0] = ~expand_nibble(fl[i] & 0xfu);
      keep[i][1] = ~expand_nibble(fl[i] >> 4);
      slot[i] = pre_s[w] + __popc(mask_s[w] & ((1u << sh) - 1u));
    }
  }
  int ok3 = 1;
  for (int c = 0; c < nch; ++c) {
    const int rb = c * H, rc = min(H, nr - rb);
    // streaming: the chunk's rows again (every thread reads all of them
    // below: its group's rows, and group 0 every row for the outlier entries)
    if (streaming && ok3 && !wait_chunk(2, c)) ok3 = 0;
    ok3 = __syncthreads_and(ok3);
    if (ok3) {
      // row maxima over the non-outlier columns (vectors past K have keep = 0),
      // four rows at a time so that their loads and reductions overlap
      for (int k0 = 0; g + RG * k0 < rc; k0 += 4) {
        uint32_t m[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = g + RG * (k0 + u);
          if (i < rc) {
            const uint4* row = xs + static_cast<size_t>(slot_of(c, i)) * nvec;
#pragma unroll
            for (int i2 = 0; i2 < VPT; ++i2) {
              const uint4 x = row[min(t + i2 * CT, nvec - 1)];
              // the byte masks widened to 16-bit lanes, with the sign bits cleared
              m[u] = __vmaxu2(m[u], x.x & __byte_perm(keep[i2][0], 0u, 0x1100) & 0x7fff7fffu);
              m[u] = __vmaxu2(m[u], x.y & __byte_perm(keep[i2][0], 0u, 0x3322) & 0x7fff7fffu);
              m[u] = __vmaxu2(m[u], x.z & __byte_perm(keep[i2][1], 0u, 0x1100) & 0x7fff7fffu);
              m[u] = __vmaxu2(m[u], x.w & __byte_perm(keep[i2][1], 0u, 0x3322) & 0x7fff7fffu);
            }
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = g + RG * (k0 + u);  // the same for the whole warp
          const uint32_t r = __reduce_max_sync(0xffffffffu, max_pair(m[u]));
          if (lane == 0 && i < rc) atomicMax(&rowmax_s[i], r);
        }
      }
      __syncthreads();
      for (int i = tid; i < rc; i += NT) {
        const float cx = scale_from_absmax_bits(rowmax_s[i]);
        c_s[i] = cx;
        a.c_x[r0 + rb + i] = cx;
        rowmax_s[i] = 0u;  // for the next chunk
      }
      __syncthreads();
      // codes (outlier columns 0)
#pragma unroll 2
      for (int i = g; i < rc; i += RG) {
        const float cx = c_s[i];
        const uint4* row = xs + static_cast<size_t>(slot_of(c, i)) * nvec;
        int8_t* qrow = a.Xq + static_cast<size_t>(r0 + rb + i) * K;
#pragma unroll
        for (int i2 = 0; i2 < VPT; ++i2) {
          const int v = t + i2 * CT;
          if (v < nvec) {
            const uint4 x = row[v];
            uint2 q = quant8_fma(x, cx);
            q.x &= keep[i2][0];
            q.y &= keep[i2][1];
            *reinterpret_cast<uint2*>(qrow + static_cast<size_t>(v) * 8) = q;
          }
        }
      }
      // the outlier entries, X_OT[o][r0 + rb + i]: the warps of row group 0
      // take the outlier vectors their lanes own, one at a time, and write
      // the chunk's rows of each outlier column with consecutive lanes on
      // consecutive rows (one coalesced store per column and 32 rows, instead
      // of a partial-sector store per entry)
      if (g == 0) {
        const __half* xh = reinterpret_cast<const __half*>(xs);
#pragma unroll
        for (int i2 = 0; i2 < VPT; ++i2) {
          uint32_t owners = __ballot_sync(0xffffffffu, fl[i2] != 0u);
          while (owners) {
            const int src = __ffs(owners) - 1;
            owners &= owners - 1;
            const uint32_t f = __shfl_sync(0xffffffffu, fl[i2], src);
            const int col0 = 8 * (__shfl_sync(0xffffffffu, t, src) + i2 * CT);
            int o = __shfl_sync(0xffffffffu, slot[i2], src);
            for (int e = 0; e < 8; ++e) {
              if ((f >> e) & 1u) {
                __half* dst = a.X_OT + static_cast<size_t>(o) * a.ld_xo + r0 + rb;
                for (int i = lane; i < rc; i += 32)
                  dst[i] = xh[static_cast<size_t>(slot_of(c, i)) * K + col0 + e];
                ++o;
              }
            }
          }
        }
      }
    }
    if (streaming) {
      __syncthreads();  // the half is free
      if (tid == 0 && ok3 && c + 2 < nch) issue(2, c + 2);
    }
  }
  if (!ok3 && tid == 0) {
    atomicOr(a.status, kStatusTimeout);
    drain();  // leave no bulk copy in flight into this block's shared memory
  }
}

struct Shape {
  int vpt, col_threads, threads;
  int64_t rows;   // per block
  int64_t chunk;  // rows per chunk (= rows when they all fit at once)
  int64_t slots;  // row slots in shared memory
};

size_t smem_bytes(int64_t slots, int64_t chunk, int64_t K) {
  const int64_t KW = (K + 31) / 32;
  return static_cast<size_t>(slots * 2 * K + KW * 8 + ((2 * chunk + 1) & ~int64_t(1)) * 4 + slots * 8);
}

Shape shape_for(int64_t M, int64_t K, int num_sms) {
  Shape s;
  const int64_t nvec = K / 8;
  s.vpt = nvec <= kMaxThreads ? 1 : nvec <= 2 * kMaxThreads ? 2 : 4;
  s.col_threads = static_cast<int>(32 * ((nvec + 32 * s.vpt - 1) / (32 * s.vpt)));
  s.rows = (M + num_sms - 1) / num_sms;
  if (s.rows <= kRowActMaxRows && smem_bytes(s.rows, s.rows, K) <= kRowActSmemMax) {
    s.chunk = s.slots = s.rows;  // every row of the block stays in shared memory
  } else {
    // streamed in chunks through two halves of the slots
    int64_t h = std::min<int64_t>(kRowActMaxRows, s.rows);
    while (h > 0 && smem_bytes(2 * h, h, K) > kRowActSmemMax) --h;
    s.chunk = h;
    s.slots = 2 * h;
  }
  const int64_t groups = std::max<int64_t>(1, std::min<int64_t>(kMaxThreads / s.col_threads, std::max<int64_t>(1, s.chunk)));
  s.threads = static_cast<int>(groups * s.col_threads);
  return s;
}

template <int VPT>
cudaError_t launch_t(const RowActArgs& a, unsigned grid, unsigned threads, size_t smem, cudaStream_t stream) {
  static unsigned long long attr_set = 0;  // one bit per device
  int dev = 0;
  cudaGetDevice(&dev);
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_set & bit)) {
    cudaError_t e = cudaFuncSetAttribute(xact_rows_kernel<VPT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kRowActSmemMax));
    if (e != cudaSuccess) return e;
    attr_set |= bit;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeCooperative;  // all blocks resident at once (grid barrier)
  attr.val.cooperative = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, xact_rows_kernel<VPT>, a);
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
  return shape_for(M, K, num_sms).chunk >= 1;
}

cudaError_t launch_row_act(const RowActArgs& args, int num_sms, cudaStream_t stream) {
  RowActArgs a = args;
  const Shape s = shape_for(a.M, a.K, num_sms);
  if (s.chunk < 1) return cudaErrorInvalidValue;
  a.rows_per_block = static_cast<int>(s.rows);
  a.chunk_rows = static_cast<int>(s.chunk);
  a.slots = static_cast<int>(s.slots);
  a.col_threads = s.col_threads;
  const unsigned grid = static_cast<unsigned>((a.M + s.rows - 1) / s.rows);
  const size_t smem = smem_bytes(s.slots, s.chunk, a.K);
  const unsigned threads = static_cast<unsigned>(s.threads);
  if (s.vpt == 1) return launch_t<1>(a, grid, threads, smem, stream);
  if (s.vpt == 2) return launch_t<2>(a, grid, threads, smem, stream);
  return launch_t<4>(a, grid, threads, smem, stream);
}

}  // namespace i8mm
