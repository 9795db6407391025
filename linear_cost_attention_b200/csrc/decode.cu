// Single-token decode step: an HBM-streaming kernel over the fp32 state.
//
// "对称性感知泰勒近似注意力机制的恒定计算成本工程实现", section "恒定计算成本的工程实现":
// per token, map k through the index tables M_p, fold it into the fixed-size
// state, and read the output as the weighted sum of every degree's
// contribution; the work is the same at any context length.  Here all degrees
// (all basis rows) are streamed in one pass: each element of
// state[B,H,m,dV+1] is read once and written once (S' = S + phi_r(k) v1_c) and
// multiplied by phi_r(q) into the per-head partial sums y[c]; the step ends
// with out = y[:dV] / y[dV].  The token attends to itself (update, then read).
//
// Access pattern: the state is one flat fp32 array of E = B*H*m*(dV+1)
// elements.  A block of NT = (dV+1)*KB threads moves 4*NT consecutive elements
// per iteration with one 16-byte load and store per thread, so every thread
// keeps the same 4 columns across iterations (4*NT is a multiple of dV+1) and
// accumulates y in registers; heads and rows come from a per-block table of
// the rows it touches.
#include <algorithm>

#include "common.cuh"
#include "sata_internal.h"

namespace sata {
namespace {

constexpr int kIters = 32;  // iterations (of 4*NT elements) per block: 32 measured
                            // 2% faster than 16 (fewer per-block feature prologues)
constexpr int kUnroll = 4;  // iterations whose loads are in flight together

template <int D1> struct DecodeShape;
template <> struct DecodeShape<65> { static constexpr int KB = 4; };   // 260 threads
template <> struct DecodeShape<33> { static constexpr int KB = 8; };   // 264
template <> struct DecodeShape<17> { static constexpr int KB = 15; };  // 255
template <> struct DecodeShape<9> { static constexpr int KB = 28; };   // 252

template <int D1, typename T>
__global__ void __launch_bounds__(D1 *DecodeShape<D1>::KB)
    decode_stream(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                  float *__restrict__ state, const uint32_t *__restrict__ idx,
                  const float *__restrict__ w, int m, int dK, long long E, float *__restrict__ y) {
  constexpr int KB = DecodeShape<D1>::KB;
  constexpr int NT = D1 * KB;
  constexpr int PER_IT = 4 * NT;
  constexpr int ROWS_IT = 4 * KB;
  constexpr long long L = (long long)PER_IT * kIters;
  constexpr int MAXROWS = ROWS_IT * kIters + 1;
  constexpr int DV = D1 - 1;
  __shared__ float s_fq[MAXROWS];
  __shared__ float s_fk[MAXROWS];
  __shared__ int s_bh[MAXROWS];
  __shared__ float s_y[2][D1];

  const int tid = threadIdx.x;
  const long long e_begin = (long long)blockIdx.x * L;
  const long long e_end = min(E, e_begin + L);
  const long long r_first = e_begin / D1;  // e_begin is a multiple of D1
  const int nrows = (int)((e_end - 1) / D1 - r_first + 1);
  const int head_first = (int)(r_first / m);

  for (int i = tid; i < nrows; i += NT) {
    const long long r = r_first + i;
    const int bh = (int)(r / m);
    const int a = (int)(r - (long long)bh * m);
    const uint32_t pk = idx[a];
    const int deg = packed_degree(pk);
    float fq = w[a], fk = fq;
    for (int s = 0; s < deg; ++s) {
      const int ii = packed_index(pk, s);
      fq *= to_f32(q[(size_t)bh * dK + ii]);
      fk *= to_f32(k[(size_t)bh * dK + ii]);
    }
    s_fq[i] = fq;
    s_fk[i] = fk;
    s_bh[i] = bh;
  }
  for (int i = tid; i < 2 * D1; i += NT) (&s_y[0][0])[i] = 0.f;
  __syncthreads();

  int col[4], rof[4], cur[4];
  float acc[4], vv[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    col[u] = (4 * tid + u) % D1;
    rof[u] = (4 * tid + u) / D1;
    cur[u] = -1;
    acc[u] = 0.f;
    vv[u] = 0.f;
  }

  auto flush = [&](int u) {
    if (cur[u] < 0) return;
    if (cur[u] == head_first)
      atomicAdd(&s_y[0][col[u]], acc[u]);
    else if (cur[u] == head_first + 1)
      atomicAdd(&s_y[1][col[u]], acc[u]);
    else
      atomicAdd(&y[(size_t)cur[u] * D1 + col[u]], acc[u]);
    acc[u] = 0.f;
  };

  // kUnroll iterations at a time: all their 16-byte loads are issued before any
  // is used, so each thread keeps kUnroll*16 bytes in flight.
  for (int it0 = 0; it0 < kIters; it0 += kUnroll) {
    float s[kUnroll][4];
    long long e[kUnroll];
#pragma unroll
    for (int j = 0; j < kUnroll; ++j) {
      e[j] = e_begin + (long long)(it0 + j) * PER_IT + 4 * tid;
      if (e[j] + 3 < e_end) {
        const float4 x = __ldcs(reinterpret_cast<const float4 *>(state + e[j]));
        s[j][0] = x.x; s[j][1] = x.y; s[j][2] = x.z; s[j][3] = x.w;
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u) s[j][u] = (e[j] + u < e_end) ? state[e[j] + u] : 0.f;
      }
    }
#pragma unroll
    for (int j = 0; j < kUnroll; ++j) {
      if (e[j] >= e_end) break;
      const bool full = (e[j] + 3 < e_end);
      const int rbase = (it0 + j) * ROWS_IT;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (!full && e[j] + u >= e_end) continue;  // past the end of the array
        const int rr = min(rbase + rof[u], nrows - 1);
        const int bh = s_bh[rr];
        if (bh != cur[u]) {
          flush(u);
          cur[u] = bh;
          vv[u] = (col[u] < DV) ? to_f32(v[(size_t)bh * DV + col[u]]) : 1.f;
        }
        const float sn = fmaf(s_fk[rr], vv[u], s[j][u]);
        s[j][u] = sn;
        acc[u] = fmaf(s_fq[rr], sn, acc[u]);
      }
      if (full) {
        __stcs(reinterpret_cast<float4 *>(state + e[j]),
               make_float4(s[j][0], s[j][1], s[j][2], s[j][3]));
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (e[j] + u < e_end) state[e[j] + u] = s[j][u];
      }
    }
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) flush(u);
  __syncthreads();
  const int head_last = s_bh[nrows - 1];
  for (int i = tid; i < 2 * D1; i += NT) {
    const int slot = i / D1, c = i % D1;
    if (head_first + slot <= head_last)
      atomicAdd(&y[(size_t)(head_first + slot) * D1 + c], s_y[slot][c]);
  }
}

template <int D1>
__global__ void decode_finalize(const float *__restrict__ y, float *__restrict__ out, int BH) {
  constexpr int DV = D1 - 1;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)BH * DV) return;
  const long long bh = i / DV, c = i % DV;
  out[i] = y[bh * D1 + c] / y[bh * D1 + DV];
}

template <int D1, typename T>
int run_decode(const void *q, const void *k, const void *v, float *state, float *out, int BH,
               int dK, const DeviceBasis *basis, cudaStream_t stream) {
  constexpr int NT = D1 * DecodeShape<D1>::KB;
  constexpr long long L = 4LL * NT * kIters;
  const long long E = (long long)BH * basis->m * D1;
  int st = SATA_OK;
  float *y = (float *)get_workspace(stream, (size_t)BH * D1 * sizeof(float), &st);
  if (!y) return st;
  cudaError_t e = cudaMemsetAsync(y, 0, (size_t)BH * D1 * sizeof(float), stream);
  if (e != cudaSuccess) return SATA_ERR_CUDA;
  const long long blocks = (E + L - 1) / L;
  if (blocks > 0x7fffffffLL) return SATA_ERR_INVALID_ARG;
  prof_kernel_begin(stream, K_DECODE_STREAM);
  decode_stream<D1, T><<<(unsigned)blocks, NT, 0, stream>>>(
      (const T *)q, (const T *)k, (const T *)v, state, basis->idx, basis->w, (int)basis->m, dK,
      E, y);
  prof_kernel_end(stream);
  const int n = BH * (D1 - 1);
  prof_kernel_begin(stream, K_DECODE_FINALIZE);
  decode_finalize<D1><<<(n + 255) / 256, 256, 0, stream>>>(y, out, BH);
  prof_kernel_end(stream);
  return cuda_status(cudaGetLastError());
}

template <typename T>
int dispatch(int dK, int dV, const void *q, const void *k, const void *v, float *state,
             float *out, int BH, const DeviceBasis *b, cudaStream_t s) {
  switch (dV) {
    case 8: return run_decode<9, T>(q, k, v, state, out, BH, dK, b, s);
    case 16: return run_decode<17, T>(q, k, v, state, out, BH, dK, b, s);
    case 32: return run_decode<33, T>(q, k, v, state, out, BH, dK, b, s);
    case 64: return run_decode<65, T>(q, k, v, state, out, BH, dK, b, s);
  }
  return SATA_ERR_UNSUPPORTED;
}

}  // namespace

int launch_decode(const void *q, const void *k, const void *v, float *state, float *out, int B,
                  int H, int dK, int dV, int P, bool bf16, const DeviceBasis *basis,
                  cudaStream_t stream) {
  (void)P;
  const int BH = B * H;
  if (bf16) return dispatch<__nv_bfloat16>(dK, dV, q, k, v, state, out, BH, basis, stream);
  return dispatch<float>(dK, dV, q, k, v, state, out, BH, basis, stream);
}

}  // namespace sata

namespace sata {
namespace {

// Same two kernels as run_decode, with the basis tables and the partial-sum
// scratch supplied by the caller instead of the library's caches.
template <int D1, typename T>
int run_decode_scratch(const void *q, const void *k, const void *v, float *state, float *out,
                       int BH, int dK, const uint32_t *idx, const float *w, int64_t m, float *y,
                       cudaStream_t stream) {
  constexpr int NT = D1 * DecodeShape<D1>::KB;
  constexpr long long L = 4LL * NT * kIters;
  const long long E = (long long)BH * m * D1;
  if (cudaMemsetAsync(y, 0, (size_t)BH * D1 * sizeof(float), stream) != cudaSuccess)
    return SATA_ERR_CUDA;
  const long long blocks = (E + L - 1) / L;
  if (blocks > 0x7fffffffLL) return SATA_ERR_INVALID_ARG;
  decode_stream<D1, T><<<(unsigned)blocks, NT, 0, stream>>>(
      (const T *)q, (const T *)k, (const T *)v, state, idx, w, (int)m, dK, E, y);
  const int n = BH * (D1 - 1);
  decode_finalize<D1><<<(n + 255) / 256, 256, 0, stream>>>(y, out, BH);
  return cuda_status(cudaGetLastError());
}

template <typename T>
int dispatch_scratch(int dK, int dV, const void *q, const void *k, const void *v, float *state,
                     float *out, int BH, const uint32_t *idx, const float *w, int64_t m,
                     float *y, cudaStream_t s) {
  switch (dV) {
    case 8: return run_decode_scratch<9, T>(q, k, v, state, out, BH, dK, idx, w, m, y, s);
    case 16: return run_decode_scratch<17, T>(q, k, v, state, out, BH, dK, idx, w, m, y, s);
    case 32: return run_decode_scratch<33, T>(q, k, v, state, out, BH, dK, idx, w, m, y, s);
    case 64: return run_decode_scratch<65, T>(q, k, v, state, out, BH, dK, idx, w, m, y, s);
  }
  return SATA_ERR_UNSUPPORTED;
}

}  // namespace

int launch_decode_scratch(const void *q, const void *k, const void *v, float *state, float *out,
                          int B, int H, int dK, int dV, bool bf16, const uint32_t *idx,
                          const float *w, int64_t m, float *y, cudaStream_t stream) {
  const int BH = B * H;
  if (bf16)
    return dispatch_scratch<__nv_bfloat16>(dK, dV, q, k, v, state, out, BH, idx, w, m, y, stream);
  return dispatch_scratch<float>(dK, dV, q, k, v, state, out, BH, idx, w, m, y, stream);
}

}  // namespace sata
