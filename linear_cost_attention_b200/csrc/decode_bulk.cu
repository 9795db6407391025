// Decode step that streams the state through shared memory with bulk async
// copies, for fp32 states and for the mixed-precision state (rows of degree
// <= 2 in fp32, rows of higher degree in fp16).
//
// "对称性感知泰勒近似注意力机制的恒定计算成本工程实现", section "恒定计算成本的工程实现":
// per token, k is mapped through the index tables M_p and folded into the
// fixed-size state, and the output is the weighted sum of every degree's
// contribution read from it; section "硬件优化路径与当前局限" notes that fp16
// storage halves the bandwidth.  Each element of the state is read once and
// written once per step (S' = S + phi_r(k) [v, 1]_c), and phi_r(q) S'_rc is
// summed into the per-head partials y[c]; out = y[:dV] / y[dV] afterwards.
//
// Why bulk copies: the step is bound by HBM bandwidth, which needs many bytes
// in flight per SM.  A thread-per-16-bytes streaming kernel keeps them in
// registers, so the bytes in flight are capped by the register file (and a
// 2-byte fp16 stream needs twice the registers for the same bytes).  Here a
// producer thread moves whole segments (16 KiB) between HBM and a ring of
// shared-memory stages with cp.async.bulk (plain bulk copies, no tensor map,
// no multicast), and the compute warps update each stage in place.
//
// Work split: the state is cut into segments of 64 fp32 rows or 128 fp16
// rows (both 256 * (dV+1) bytes, 16-byte aligned because every array starts
// 16-byte aligned and a segment is a multiple of 16 bytes); each CTA owns a
// contiguous range of segments, so the head of its rows changes rarely and
// the partials stay in registers.  Rows past the last full segment of each
// array (the tails) are updated in global memory by the grid's last CTA.
#include <cuda_fp16.h>

#include <algorithm>

#include "common.cuh"
#include "sata_internal.h"
#include "tc_common.cuh"

namespace sata {
namespace {

using namespace tc;

constexpr int kStages = 3;     // shared-memory ring
constexpr int kLag = 2;        // segment i's store is issued after segment i + kLag's load
constexpr int kCtasPerSm = 4;  // 4 x 50 KiB of ring per SM (dV = 64); measured against
                               // 3 x 4 stages (10% slower) and 2 x 5 stages (45% slower)
constexpr int kRows32 = 64;    // rows per fp32 segment
constexpr int kRows16 = 128;   // rows per fp16 segment

template <int D1> struct BulkShape;
template <> struct BulkShape<65> { static constexpr int KB = 4; };  // 260 compute threads
template <> struct BulkShape<33> { static constexpr int KB = 8; };  // 264

struct BulkParams {
  float *lo;        // [BH][m_lo][D1] fp32 rows (all rows for an fp32 state)
  __half *hi;       // [BH][m_hi][D1] fp16 rows of the mixed state (null if m_hi == 0)
  int m_lo, m_hi;   // rows per head in each array
  long long rows_lo, rows_hi;   // BH * m_lo, BH * m_hi
  long long nseg_lo, nseg_hi;   // full segments in each array
  const uint32_t *idx;          // packed basis rows (common.cuh)
  const float *w;               // basis weights
  int dK;
  float *y;                     // [BH][D1] partial sums, zeroed by the caller
  int *err;
  long long wait_limit;
};

__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes,
                                          uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void bulk_store(void *dst, const void *src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
               "r"(smem_u32(src)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// At most N of this thread's committed store groups still read shared memory.
template <int N> __device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Every committed store group of this thread has completed.
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Named barrier over the compute warps that also ANDs a predicate across
// them, so that every compute thread takes the same stop decision.
__device__ __forceinline__ bool bar_and(int id, int nthreads, bool pred) {
  int r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.b32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((int)pred), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

// phi_r(q), phi_r(k) and the head of global row `row` of one array.
template <typename T>
__device__ __forceinline__ float4 row_meta(const T *q, const T *k, const BulkParams &p,
                                           long long row, bool hi) {
  const int m = hi ? p.m_hi : p.m_lo;
  const int h = (int)(row / m);
  const int a = (int)(row - (long long)h * m) + (hi ? p.m_lo : 0);
  const uint32_t pk = p.idx[a];
  const int deg = packed_degree(pk);
  float fq = p.w[a], fk = fq;
  for (int s = 0; s < deg; ++s) {
    const int ii = packed_index(pk, s);
    fq *= to_f32(q[(size_t)h * p.dK + ii]);
    fk *= to_f32(k[(size_t)h * p.dK + ii]);
  }
  return make_float4(fq, fk, __int_as_float(h), 0.f);
}

template <int D1, typename T>
__global__ void __launch_bounds__((D1 * BulkShape<D1>::KB + 31) / 32 * 32 + 32)
    decode_bulk(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                const BulkParams p) {
  constexpr int KB = BulkShape<D1>::KB;
  constexpr int NT = D1 * KB;         // compute threads doing element work
  constexpr int NW = (NT + 31) / 32;  // compute warps (the last one partly idle)
  constexpr int DV = D1 - 1;
  constexpr uint32_t SB = 256u * D1;  // segment bytes (64 fp32 or 128 fp16 rows)
  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ uint64_t full[kStages], done[kStages];
  __shared__ float4 meta[2][kRows16];
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long nseg = p.nseg_lo + p.nseg_hi;
  const long long s_begin = (long long)blockIdx.x * nseg / gridDim.x;
  const long long s_end = (long long)(blockIdx.x + 1) * nseg / gridDim.x;
  const int n = (int)(s_end - s_begin);
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&done[s], NW);
    }
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  auto seg_gmem = [&](long long s) -> uint8_t * {
    return s < p.nseg_lo ? reinterpret_cast<uint8_t *>(p.lo + s * kRows32 * D1)
                         : reinterpret_cast<uint8_t *>(p.hi + (s - p.nseg_lo) * kRows16 * D1);
  };

  if (warp == NW) {
    // ---------------- producer: bulk loads into the ring, bulk stores back
    if (lane == 0) {
      bool ok = true;
      int loads = 0;
      for (int i = 0; ok && i < n + kLag; ++i) {
        if (i < n) {
          const int st = i % kStages;
          // stores issued so far: segments < i - kLag; the one of segment
          // i - kStages must have finished reading this stage
          if (i >= kStages) bulk_wait_read<kStages - 1 - kLag>();
          mbar_arrive_expect_tx(&full[st], SB);
          bulk_load(ring + st * SB, seg_gmem(s_begin + i), SB, &full[st]);
          ++loads;
        }
        const int j = i - kLag;
        if (j >= 0 && j < n) {
          ok = mbar_wait(&done[j % kStages], (j / kStages) & 1, &abort_flag, p.err, p.wait_limit);
          if (!ok) break;
          bulk_store(seg_gmem(s_begin + j), ring + (j % kStages) * SB, SB);
          bulk_commit();
        }
      }
      bulk_wait_all();  // every store has landed
      // every load this CTA issued has landed before the ring goes away
      for (int j = std::max(0, loads - kStages); j < loads; ++j) {
        volatile int never = 0;
        mbar_wait(&full[j % kStages], (j / kStages) & 1, &never, p.err);
      }
    }
  } else {
    // ---------------- compute warps
    const bool worker = tid < NT;
    const int c = tid % D1, ro = tid / D1;
    int cur = -1;
    float acc = 0.f, vc = 0.f;
    auto flush = [&]() {
      if (cur >= 0) atomicAdd(&p.y[(size_t)cur * D1 + c], acc);
      acc = 0.f;
    };
    auto use_head = [&](int h) {
      if (h != cur) {
        flush();
        cur = h;
        vc = c < DV ? to_f32(v[(size_t)h * DV + c]) : 1.f;
      }
    };
    bool ok = true;
    for (int i = 0; i < n; ++i) {
      const long long s = s_begin + i;
      const bool hi = s >= p.nseg_lo;
      const int slot = i & 1;
      const long long r0 = hi ? (s - p.nseg_lo) * kRows16 : s * kRows32;
      if (tid < (hi ? kRows16 : kRows32)) meta[slot][tid] = row_meta(q, k, p, r0 + tid, hi);
      // publishes meta[slot]; every thread has finished segment i - 1 (and so
      // no longer reads meta[slot] of segment i - 2)
      if (!bar_and(1, NW * 32, ok)) break;
      const int st = i % kStages;
      ok = mbar_wait(&full[st], (i / kStages) & 1, &abort_flag, p.err, p.wait_limit);
      if (!ok) continue;  // the next barrier stops every compute thread
      if (worker) {
        // a segment inside one head (all but a few) takes the loops without
        // a per-row head check; y takes the updated value before it is
        // rounded to the stored precision
        const int rows = hi ? kRows16 : kRows32;
        const int h0 = __float_as_int(meta[slot][0].z);
        const bool one_head = h0 == __float_as_int(meta[slot][rows - 1].z);
        if (one_head) use_head(h0);
        const float2 *mq = reinterpret_cast<const float2 *>(meta[slot]);  // (phi_q, phi_k) per row
        if (hi) {
          __half *sg = reinterpret_cast<__half *>(ring + st * SB);
          if (one_head) {
#pragma unroll 8
            for (int j = 0; j < kRows16 / KB; ++j) {
              const int rl = ro + KB * j;
              const float2 mt = mq[2 * rl];
              const int e = rl * D1 + c;
              const float sn = fmaf(mt.y, vc, __half2float(sg[e]));
              sg[e] = __float2half_rn(sn);
              acc = fmaf(mt.x, sn, acc);
            }
          } else {
#pragma unroll 4
            for (int j = 0; j < kRows16 / KB; ++j) {
              const int rl = ro + KB * j;
              const float4 mt = meta[slot][rl];
              use_head(__float_as_int(mt.z));
              const int e = rl * D1 + c;
              const float sn = fmaf(mt.y, vc, __half2float(sg[e]));
              sg[e] = __float2half_rn(sn);
              acc = fmaf(mt.x, sn, acc);
            }
          }
        } else {
          float *sg = reinterpret_cast<float *>(ring + st * SB);
          if (one_head) {
#pragma unroll 8
            for (int j = 0; j < kRows32 / KB; ++j) {
              const int rl = ro + KB * j;
              const float2 mt = mq[2 * rl];
              const int e = rl * D1 + c;
              const float sn = fmaf(mt.y, vc, sg[e]);
              sg[e] = sn;
              acc = fmaf(mt.x, sn, acc);
            }
          } else {
#pragma unroll 4
            for (int j = 0; j < kRows32 / KB; ++j) {
              const int rl = ro + KB * j;
              const float4 mt = meta[slot][rl];
              use_head(__float_as_int(mt.z));
              const int e = rl * D1 + c;
              const float sn = fmaf(mt.y, vc, sg[e]);
              sg[e] = sn;
              acc = fmaf(mt.x, sn, acc);
            }
          }
        }
      }
      fence_proxy_async_smem();  // these writes are read next by the bulk store
      __syncwarp();
      if (lane == 0) mbar_arrive(&done[st]);
    }
    if (worker) flush();
  }
  __syncthreads();

  // ---------------- tails: rows past the last full segment, in global memory
  if (blockIdx.x == gridDim.x - 1 && warp < NW) {
    for (int part = 0; part < 2; ++part) {
      const bool hi = part == 1;
      const long long first = hi ? p.nseg_hi * kRows16 : p.nseg_lo * kRows32;
      const long long rows = hi ? p.rows_hi : p.rows_lo;
      const long long ne = (rows - first) * D1;
      for (long long e = tid; e < ne; e += NW * 32) {
        const long long row = first + e / D1;
        const int cc = (int)(e % D1);
        const float4 mt = row_meta(q, k, p, row, hi);
        const int h = __float_as_int(mt.z);
        const float vv = cc < DV ? to_f32(v[(size_t)h * DV + cc]) : 1.f;
        const size_t g = (size_t)row * D1 + cc;
        float sn;
        if (hi) {
          const __half hn = __float2half_rn(fmaf(mt.y, vv, __half2float(p.hi[g])));
          p.hi[g] = hn;
          sn = __half2float(hn);
        } else {
          sn = fmaf(mt.y, vv, p.lo[g]);
          p.lo[g] = sn;
        }
        atomicAdd(&p.y[(size_t)h * D1 + cc], mt.x * sn);
      }
    }
  }
}

template <int D1>
__global__ void bulk_finalize(const float *__restrict__ y, float *__restrict__ out, int BH) {
  constexpr int DV = D1 - 1;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)BH * DV) return;
  const long long bh = i / DV, c = i % DV;
  out[i] = y[bh * D1 + c] / y[bh * D1 + DV];
}

template <int D1, typename T>
int run_bulk(const void *q, const void *k, const void *v, float *lo, __half *hi, int BH, int dK,
             int m_lo, int m_hi, const DeviceBasis *basis, float *out, cudaStream_t stream) {
  constexpr int NT = D1 * BulkShape<D1>::KB;
  constexpr int threads = (NT + 31) / 32 * 32 + 32;
  constexpr uint32_t SB = 256u * D1;
  constexpr size_t smem = (size_t)kStages * SB;
  int st = SATA_OK;
  float *y = (float *)get_workspace(stream, (size_t)BH * D1 * sizeof(float), &st);
  if (!y) return st;
  if (cudaMemsetAsync(y, 0, (size_t)BH * D1 * sizeof(float), stream) != cudaSuccess)
    return SATA_ERR_CUDA;
  BulkParams p;
  p.lo = lo;
  p.hi = hi;
  p.m_lo = m_lo;
  p.m_hi = m_hi;
  p.rows_lo = (long long)BH * m_lo;
  p.rows_hi = (long long)BH * m_hi;
  p.nseg_lo = p.rows_lo / kRows32;
  p.nseg_hi = p.rows_hi / kRows16;
  p.idx = basis->idx;
  p.w = basis->w;
  p.dK = dK;
  p.y = y;
  p.err = device_error_ptr();
  if (!p.err) return SATA_ERR_NOMEM;
  p.wait_limit = tc_wait_limit();
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (cudaFuncSetAttribute(decode_bulk<D1, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return SATA_ERR_CUDA;
  const long long nseg = p.nseg_lo + p.nseg_hi;
  const int grid = (int)std::max<long long>(1, std::min<long long>(nseg, (long long)nsm * kCtasPerSm));
  prof_kernel_begin(stream, K_DECODE_BULK);
  decode_bulk<D1, T><<<grid, threads, smem, stream>>>((const T *)q, (const T *)k, (const T *)v, p);
  prof_kernel_end(stream);
  const int nout = BH * (D1 - 1);
  prof_kernel_begin(stream, K_DECODE_FINALIZE);
  bulk_finalize<D1><<<(nout + 255) / 256, 256, 0, stream>>>(y, out, BH);
  prof_kernel_end(stream);
  return cuda_status(cudaGetLastError());
}

// state [BH][m][D1] fp32 <-> mixed (lo [BH][m_lo][D1] fp32, hi [BH][m - m_lo][D1] fp16)
__global__ void state_split_kernel(const float *__restrict__ state, float *__restrict__ lo,
                                   __half *__restrict__ hi, long long BH, int m, int m_lo,
                                   int D1) {
  const long long per_head = (long long)m * D1, lo_head = (long long)m_lo * D1;
  const long long n = BH * per_head;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (long long)gridDim.x * blockDim.x) {
    const long long h = e / per_head, r = e - h * per_head;
    if (r < lo_head)
      lo[h * lo_head + r] = state[e];
    else
      hi[h * (per_head - lo_head) + (r - lo_head)] = __float2half_rn(state[e]);
  }
}

__global__ void state_join_kernel(const float *__restrict__ lo, const __half *__restrict__ hi,
                                  float *__restrict__ state, long long BH, int m, int m_lo,
                                  int D1) {
  const long long per_head = (long long)m * D1, lo_head = (long long)m_lo * D1;
  const long long n = BH * per_head;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (long long)gridDim.x * blockDim.x) {
    const long long h = e / per_head, r = e - h * per_head;
    state[e] = r < lo_head ? lo[h * lo_head + r]
                           : __half2float(hi[h * (per_head - lo_head) + (r - lo_head)]);
  }
}

}  // namespace

int launch_state_convert(bool split, float *state, float *lo, void *hi, long long BH, int m,
                         int m_lo, int D1, cudaStream_t stream) {
  const long long n = BH * (long long)m * D1;
  const int grid = (int)std::min<long long>((n + 255) / 256, 148LL * 16);
  if (split)
    state_split_kernel<<<grid, 256, 0, stream>>>(state, lo, reinterpret_cast<__half *>(hi), BH,
                                                 m, m_lo, D1);
  else
    state_join_kernel<<<grid, 256, 0, stream>>>(lo, reinterpret_cast<const __half *>(hi), state,
                                                BH, m, m_lo, D1);
  return cuda_status(cudaGetLastError());
}

bool bulk_decode_supported(int dV) { return dV == 64 || dV == 32; }

int launch_decode_bulk(const void *q, const void *k, const void *v, float *lo, void *hi, int B,
                       int H, int dK, int dV, int m_lo, int m_hi, bool bf16,
                       const DeviceBasis *basis, float *out, cudaStream_t stream) {
  const int BH = B * H;
  __half *h = reinterpret_cast<__half *>(hi);
  if (dV == 64)
    return bf16 ? run_bulk<65, __nv_bfloat16>(q, k, v, lo, h, BH, dK, m_lo, m_hi, basis, out, stream)
                : run_bulk<65, float>(q, k, v, lo, h, BH, dK, m_lo, m_hi, basis, out, stream);
  if (dV == 32)
    return bf16 ? run_bulk<33, __nv_bfloat16>(q, k, v, lo, h, BH, dK, m_lo, m_hi, basis, out, stream)
                : run_bulk<33, float>(q, k, v, lo, h, BH, dK, m_lo, m_hi, basis, out, stream);
  return SATA_ERR_UNSUPPORTED;
}

}  // namespace sata
