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

constexpr int kIters = 16;  // iterations (of 4*NT elements) per block
constexpr int kUnroll = 4;  // iterations whose loads are in flight together

template <int D1> struct DecodeShape;
template <> struct DecodeShape<65> { static constexpr int KB = 4; };   // 260 threads
template <> struct DecodeShape<33> { static constexpr int KB = 8; };   // 264
template <> struct DecodeShape<17> { static constexpr int KB = 15; };  // 255
template <> struct DecodeShape<9> { static constexpr int KB = 28; };   // 252

template <int D1, typename T>
__global__ void __launch_bounds__(D1 *DecodeShape<D1>::KB, 3)
    decode_stream(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                  float *__restrict__ state, const uint32_t *__restrict__ idx,
                  const float *__restrict__ w, int m, int dK, long long E, float *__restrict__ y) {
  constexpr int KB = DecodeShape<D1>::KB;
  constexpr int NT = D1 * KB;
  constexpr int PER_IT = 4 * NT;
  constexpr int ROWS_IT = 4 * KB;
  constexpr long long L = (long long)PER_IT * kIters;
  constexpr int MAXROWS = ROWS_IT * kIters + 2;
  constexpr int DV = D1 - 1;
  __shared__ float2 s_f[MAXROWS];  // (phi_r(q), phi_r(k)) of the rows this block touches
  __shared__ float s_y[2][D1];

  const int tid = threadIdx.x;
  const long long e_begin = (long long)blockIdx.x * L;
  const long long e_end = min(E, e_begin + L);
  const long long r_first = e_begin / D1;  // e_begin is a multiple of D1
  const int nrows = (int)((e_end - 1) / D1 - r_first + 1);
  const int head_first = (int)(r_first / m);
  const int head_last = (int)(((e_end - 1) / D1) / m);
  // first block-relative row of the second head (beyond the block if none)
  const int split_row = (int)min((long long)MAXROWS, (long long)(head_first + 1) * m - r_first);

  for (int i = tid; i < nrows; i += NT) {
    const long long r = r_first + i;
    const int bh = (int)(r / m);
    const int a = (int)(r - (long long)bh * m);
    const uint32_t pk = idx[a];
    const int deg = pk >> 24;
    float fq = w[a], fk = fq;
    for (int s = 0; s < deg; ++s) {
      const int ii = (pk >> (8 * s)) & 0xff;
      fq *= to_f32(q[(size_t)bh * dK + ii]);
      fk *= to_f32(k[(size_t)bh * dK + ii]);
    }
    s_f[i] = make_float2(fq, fk);
  }
  if (tid < 2) s_f[nrows + tid] = make_float2(0.f, 0.f);
  for (int i = tid; i < 2 * D1; i += NT) (&s_y[0][0])[i] = 0.f;
  __syncthreads();

  // this thread's 4 elements of every iteration: fixed columns, rows rof0 or
  // rof0 + 1 (element u sits in the second row when u >= usplit)
  int col[4];
  const int rof0 = (4 * tid) / D1;
  int usplit = 4;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    col[u] = (4 * tid + u) % D1;
    if (usplit == 4 && (4 * tid + u) / D1 != rof0) usplit = u;
  }
  float acc0[4], acc1[4], vv0[4], vv1[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    acc0[u] = 0.f;
    acc1[u] = 0.f;
    vv0[u] = (col[u] < DV) ? to_f32(v[(size_t)head_first * DV + col[u]]) : 1.f;
    vv1[u] = (col[u] < DV && head_first + 1 <= head_last)
                 ? to_f32(v[(size_t)(head_first + 1) * DV + col[u]])
                 : 1.f;
  }
  // rows of a third or later head (blocks that span more than two heads, only
  // when m is small) take the general path below
  const bool simple = head_last <= head_first + 1;

  for (int it0 = 0; it0 < kIters; it0 += kUnroll) {
    float sv[kUnroll][4];
    long long e[kUnroll];
#pragma unroll
    for (int j = 0; j < kUnroll; ++j) {
      e[j] = e_begin + (long long)(it0 + j) * PER_IT + 4 * tid;
      if (e[j] + 3 < e_end) {
        const float4 x = __ldcs(reinterpret_cast<const float4 *>(state + e[j]));
        sv[j][0] = x.x; sv[j][1] = x.y; sv[j][2] = x.z; sv[j][3] = x.w;
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u) sv[j][u] = (e[j] + u < e_end) ? state[e[j] + u] : 0.f;
      }
    }
#pragma unroll
    for (int j = 0; j < kUnroll; ++j) {
      if (e[j] >= e_end) break;
      const bool full = (e[j] + 3 < e_end);
      const int r0 = (it0 + j) * ROWS_IT + rof0;
      const float2 f0 = s_f[r0], f1 = s_f[r0 + 1];
      if (simple) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (!full && e[j] + u >= e_end) continue;  // past the end of the array
          const int rr = u < usplit ? r0 : r0 + 1;
          const float2 f = u < usplit ? f0 : f1;
          const bool second = rr >= split_row;
          const float sn = fmaf(f.y, second ? vv1[u] : vv0[u], sv[j][u]);
          sv[j][u] = sn;
          if (second)
            acc1[u] = fmaf(f.x, sn, acc1[u]);
          else
            acc0[u] = fmaf(f.x, sn, acc0[u]);
        }
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (!full && e[j] + u >= e_end) continue;
          const int rr = u < usplit ? r0 : r0 + 1;
          const float2 f = u < usplit ? f0 : f1;
          const int bh = (int)((r_first + rr) / m);
          const float vu = (col[u] < DV) ? to_f32(v[(size_t)bh * DV + col[u]]) : 1.f;
          const float sn = fmaf(f.y, vu, sv[j][u]);
          sv[j][u] = sn;
          const float contrib = f.x * sn;
          if (bh == head_first)
            acc0[u] += contrib;
          else if (bh == head_first + 1)
            acc1[u] += contrib;
          else
            atomicAdd(&y[(size_t)bh * D1 + col[u]], contrib);
        }
      }
      if (full) {
        __stcs(reinterpret_cast<float4 *>(state + e[j]),
               make_float4(sv[j][0], sv[j][1], sv[j][2], sv[j][3]));
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (e[j] + u < e_end) state[e[j] + u] = sv[j][u];
      }
    }
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    atomicAdd(&s_y[0][col[u]], acc0[u]);
    atomicAdd(&s_y[1][col[u]], acc1[u]);
  }
  __syncthreads();
  for (int i = tid; i < 2 * D1; i += NT) {
    const int slot = i / D1, c = i % D1;
    if (head_first + slot <= head_last)
      atomicAdd(&y[(size_t)(head_first + slot) * D1 + c], s_y[slot][c]);
  }
}

template <int D1>
__global__ void decode_finalize(const float *__restrict__ y, float *__restrict__ out, int BH) {
  constexpr int DV = D1 - 1;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= BH * DV) return;
  const int bh = i / DV, c = i % DV;
  out[i] = y[(size_t)bh * D1 + c] / y[(size_t)bh * D1 + DV];
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
