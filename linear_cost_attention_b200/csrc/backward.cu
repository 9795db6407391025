// Backward pass of causal SATA attention on CUDA cores (fp32 arithmetic).
//
// "对称感知泰勒近似实现恒定Token成本注意力机制" (ai-stack.site), FAQ 5: models are
// trained from scratch with the method, which needs the gradients of the
// attention output.  With L = sum(dout * out), out_i = num_i / den_i,
// num_i = sum_{j<=i} T_ij v_j, den_i = sum_{j<=i} T_ij, T_ij = T_P(s_ij),
// s_ij = q_i . k_j / sqrt(dK), the chain rule gives
//     dnum_i = dout_i / den_i,   dden_i = -(dout_i . out_i) / den_i,
//     dT_ij  = dnum_i . v_j + dden_i,   ds_ij = dT_ij T_{P-1}(s_ij),
//     dq_i = sum_{j<=i} ds_ij k_j / sqrt(dK),   dk_j = sum_{i>=j} ds_ij q_i / sqrt(dK),
//     dv_j = sum_{i>=j} T_ij dnum_i
// (d/ds of sum_{p<P} s^p/p! is sum_{p<P-1} s^p/p!).  These are evaluated
// exactly as written, over (query, key) tiles, so the cost is quadratic in N:
//   bwd_rows  one block per 32 queries: pass 1 over the keys j <= i gives num,
//             den, hence g_i = [dnum_i, dden_i] (stored for bwd_cols); pass 2
//             gives dq_i.
//   bwd_cols  one block per 32 keys: over the queries i >= j, dk_j and dv_j.
// All tiles are 32 x 32 (query x key) with 256 threads; inputs are widened to
// fp32 in shared memory.
#include "common.cuh"
#include "sata_internal.h"

namespace sata {
namespace {

constexpr int kBT = 32;        // queries (rows) and keys (columns) per tile
constexpr int kBThreads = 256;

// d/ds T_P(s) = T_{P-1}(s), which is 0 for P = 1 (T_1 = 1 is constant).
__device__ __forceinline__ float taylor_deriv(float s, int P) {
  return P >= 2 ? taylor_trunc(s, P - 1) : 0.f;
}

// Score tile s[r][c] = x_r . y_c (32 x 32, inner size D) into smem; each thread
// computes a 2 x 2 block.
template <int D>
__device__ __forceinline__ void score_tile(const float (&x)[kBT][D + 1], const float (&y)[kBT][D + 1],
                                           float (&s)[kBT][kBT + 1]) {
  const int t = threadIdx.x;
  const int r0 = 2 * (t >> 4), c0 = 2 * (t & 15);
  float a00 = 0.f, a01 = 0.f, a10 = 0.f, a11 = 0.f;
#pragma unroll 8
  for (int d = 0; d < D; ++d) {
    const float x0 = x[r0][d], x1 = x[r0 + 1][d], y0 = y[c0][d], y1 = y[c0 + 1][d];
    a00 = fmaf(x0, y0, a00);
    a01 = fmaf(x0, y1, a01);
    a10 = fmaf(x1, y0, a10);
    a11 = fmaf(x1, y1, a11);
  }
  s[r0][c0] = a00;
  s[r0][c0 + 1] = a01;
  s[r0 + 1][c0] = a10;
  s[r0 + 1][c0 + 1] = a11;
}

// acc[r][c] += sum_j m[r][j] * z[j][c] for c < C, for the (row, column) pairs
// of this thread: row t / 8, columns t % 8 + 8 e (e < PER).
template <int C, int PER, int ZS>
__device__ __forceinline__ void accumulate(const float (&m)[kBT][kBT + 1], const float (&z)[kBT][ZS],
                                           float (&acc)[PER]) {
  const int r = threadIdx.x >> 3, c0 = threadIdx.x & 7;
#pragma unroll 4
  for (int j = 0; j < kBT; ++j) {
    const float mv = m[r][j];
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      const int c = c0 + 8 * e;
      if (c < C) acc[e] = fmaf(mv, z[j][c], acc[e]);
    }
  }
}

// Rows row0 .. row0 + 31 of a [N, D] array, widened to fp32 (zeros past N).
template <int D, typename T>
__device__ __forceinline__ void load_rows(float (&dst)[kBT][D + 1], const T *src, int row0, int N) {
  for (int e = threadIdx.x; e < kBT * D; e += kBThreads) {
    const int r = e / D, c = e % D;
    dst[r][c] = row0 + r < N ? to_f32(src[(size_t)(row0 + r) * D + c]) : 0.f;
  }
}

// Rows row0 .. row0 + 31 of [V, 1] (V is [N, DV]), widened to fp32.
template <int DV, typename T>
__device__ __forceinline__ void load_v1(float (&dst)[kBT][DV + 2], const T *v, int row0, int N) {
  constexpr int D1 = DV + 1;
  for (int e = threadIdx.x; e < kBT * D1; e += kBThreads) {
    const int r = e / D1, c = e % D1;
    dst[r][c] = row0 + r < N ? (c < DV ? to_f32(v[(size_t)(row0 + r) * DV + c]) : 1.f) : 0.f;
  }
}

// One block per (32 queries, head).
template <int DK, int DV, typename T>
__global__ void __launch_bounds__(kBThreads)
    bwd_rows(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
             const float *__restrict__ dout, float *__restrict__ g, float *__restrict__ dq, int N,
             int P, float scale) {
  constexpr int D1 = DV + 1;
  constexpr int PV = (D1 + 7) / 8, PK = (DK + 7) / 8;
  __shared__ float qs[kBT][DK + 1], ks[kBT][DK + 1], vs[kBT][D1 + 1], gs[kBT][D1 + 1];
  __shared__ float st[kBT][kBT + 1];
  const size_t bh = blockIdx.y;
  const int i0 = blockIdx.x * kBT;
  const T *qh = q + bh * N * DK, *kh = k + bh * N * DK, *vh = v + bh * N * DV;
  load_rows<DK>(qs, qh, i0, N);
  const int r = threadIdx.x >> 3, c0 = threadIdx.x & 7;

  // pass 1: [num, den]_i = sum_{j<=i} T_ij [v_j, 1]
  float acc[PV];
#pragma unroll
  for (int e = 0; e < PV; ++e) acc[e] = 0.f;
  for (int j0 = 0; j0 <= i0 && j0 < N; j0 += kBT) {
    __syncthreads();
    load_rows<DK>(ks, kh, j0, N);
    load_v1<DV>(vs, vh, j0, N);
    __syncthreads();
    score_tile<DK>(qs, ks, st);
    __syncthreads();
    for (int e = threadIdx.x; e < kBT * kBT; e += kBThreads) {
      const int rr = e / kBT, c = e % kBT;
      st[rr][c] = (j0 + c <= i0 + rr && j0 + c < N) ? taylor_trunc(st[rr][c] * scale, P) : 0.f;
    }
    __syncthreads();
    accumulate<D1, PV, D1 + 1>(st, vs, acc);
  }
  // g_i = [dout_i / den_i, -(dout_i . out_i) / den_i]
  __syncthreads();
#pragma unroll
  for (int e = 0; e < PV; ++e) {
    const int c = c0 + 8 * e;
    if (c < D1) gs[r][c] = acc[e];  // [num, den] for now
  }
  __syncthreads();
  if (threadIdx.x < kBT) {
    const int rr = threadIdx.x, i = i0 + rr;
    if (i < N) {
      const float den = gs[rr][DV];
      float dot = 0.f;
      for (int c = 0; c < DV; ++c) dot = fmaf(dout[(bh * N + i) * DV + c], gs[rr][c] / den, dot);
      for (int c = 0; c < DV; ++c) gs[rr][c] = dout[(bh * N + i) * DV + c] / den;
      gs[rr][DV] = -dot / den;
    } else {
      for (int c = 0; c < D1; ++c) gs[rr][c] = 0.f;
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < kBT * D1; e += kBThreads) {
    const int rr = e / D1, c = e % D1;
    if (i0 + rr < N) g[(bh * N + i0 + rr) * D1 + c] = gs[rr][c];
  }

  // pass 2: dq_i = sum_{j<=i} (g_i . [v_j, 1]) T_{P-1}(s_ij) k_j * scale
  float aq[PK];
#pragma unroll
  for (int e = 0; e < PK; ++e) aq[e] = 0.f;
  for (int j0 = 0; j0 <= i0 && j0 < N; j0 += kBT) {
    __syncthreads();
    load_rows<DK>(ks, kh, j0, N);
    load_v1<DV>(vs, vh, j0, N);
    __syncthreads();
    score_tile<DK>(qs, ks, st);
    __syncthreads();
    // dT = g . [v, 1] into a second tile, then ds = dT * T_{P-1}(s)
    for (int e = threadIdx.x; e < kBT * kBT; e += kBThreads) {
      const int rr = e / kBT, c = e % kBT;
      float dT = 0.f;
#pragma unroll 8
      for (int d = 0; d < D1; ++d) dT = fmaf(gs[rr][d], vs[c][d], dT);
      const bool live = j0 + c <= i0 + rr && j0 + c < N;
      st[rr][c] = live ? dT * taylor_deriv(st[rr][c] * scale, P) : 0.f;
    }
    __syncthreads();
    accumulate<DK, PK, DK + 1>(st, ks, aq);
  }
  if (i0 + r < N) {
#pragma unroll
    for (int e = 0; e < PK; ++e) {
      const int c = c0 + 8 * e;
      if (c < DK) dq[(bh * N + i0 + r) * DK + c] = aq[e] * scale;
    }
  }
}

// One block per (32 keys, head): dk_j and dv_j over the queries i >= j.
template <int DK, int DV, typename T>
__global__ void __launch_bounds__(kBThreads)
    bwd_cols(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
             const float *__restrict__ g, float *__restrict__ dk, float *__restrict__ dv, int N,
             int P, float scale) {
  constexpr int D1 = DV + 1;
  constexpr int PV = (DV + 7) / 8, PK = (DK + 7) / 8;
  __shared__ float ks[kBT][DK + 1], qs[kBT][DK + 1], vs[kBT][D1 + 1], gs[kBT][D1 + 1];
  __shared__ float tt[kBT][kBT + 1], ds[kBT][kBT + 1];
  const size_t bh = blockIdx.y;
  const int j0 = blockIdx.x * kBT;
  const T *qh = q + bh * N * DK, *kh = k + bh * N * DK, *vh = v + bh * N * DV;
  load_rows<DK>(ks, kh, j0, N);
  load_v1<DV>(vs, vh, j0, N);
  const int r = threadIdx.x >> 3, c0 = threadIdx.x & 7;
  float ak[PK], av[PV];
#pragma unroll
  for (int e = 0; e < PK; ++e) ak[e] = 0.f;
#pragma unroll
  for (int e = 0; e < PV; ++e) av[e] = 0.f;
  for (int i0 = j0 - j0 % kBT; i0 < N; i0 += kBT) {
    __syncthreads();
    load_rows<DK>(qs, qh, i0, N);
    for (int e = threadIdx.x; e < kBT * D1; e += kBThreads) {
      const int rr = e / D1, c = e % D1;
      gs[rr][c] = i0 + rr < N ? g[(bh * N + i0 + rr) * D1 + c] : 0.f;
    }
    __syncthreads();
    score_tile<DK>(ks, qs, tt);  // tt[key][query] = s
    __syncthreads();
    for (int e = threadIdx.x; e < kBT * kBT; e += kBThreads) {
      const int kj = e / kBT, qi = e % kBT;
      const bool live = j0 + kj <= i0 + qi && i0 + qi < N && j0 + kj < N;
      const float s = tt[kj][qi] * scale;
      float dT = 0.f;
#pragma unroll 8
      for (int d = 0; d < D1; ++d) dT = fmaf(gs[qi][d], vs[kj][d], dT);
      ds[kj][qi] = live ? dT * taylor_deriv(s, P) : 0.f;
      tt[kj][qi] = live ? taylor_trunc(s, P) : 0.f;
    }
    __syncthreads();
    accumulate<DK, PK, DK + 1>(ds, qs, ak);  // dk_j += sum_i ds_ij q_i
    accumulate<DV, PV, D1 + 1>(tt, gs, av);  // dv_j += sum_i T_ij dnum_i (g's first dV columns)
  }
  if (j0 + r < N) {
#pragma unroll
    for (int e = 0; e < PK; ++e) {
      const int c = c0 + 8 * e;
      if (c < DK) dk[(bh * N + j0 + r) * DK + c] = ak[e] * scale;
    }
#pragma unroll
    for (int e = 0; e < PV; ++e) {
      const int c = c0 + 8 * e;
      if (c < DV) dv[(bh * N + j0 + r) * DV + c] = av[e];
    }
  }
}

template <int DK, int DV, typename T>
int run_backward(const void *q, const void *k, const void *v, const float *dout, float *dq,
                 float *dk, float *dv, int BH, int N, int P, cudaStream_t stream) {
  int st = SATA_OK;
  float *g = (float *)get_workspace(stream, (size_t)BH * N * (DV + 1) * sizeof(float), &st);
  if (!g) return st;
  const dim3 grid((N + kBT - 1) / kBT, BH);
  const float scale = 1.0f / sqrtf((float)DK);
  prof_kernel_begin(stream, K_BWD_ROWS);
  bwd_rows<DK, DV, T><<<grid, kBThreads, 0, stream>>>((const T *)q, (const T *)k, (const T *)v,
                                                      dout, g, dq, N, P, scale);
  prof_kernel_end(stream);
  prof_kernel_begin(stream, K_BWD_COLS);
  bwd_cols<DK, DV, T><<<grid, kBThreads, 0, stream>>>((const T *)q, (const T *)k, (const T *)v, g,
                                                      dk, dv, N, P, scale);
  prof_kernel_end(stream);
  return cuda_status(cudaGetLastError());
}

template <int DK, typename T>
int dispatch_dv(int dV, const void *q, const void *k, const void *v, const float *dout, float *dq,
                float *dk, float *dv, int BH, int N, int P, cudaStream_t s) {
  switch (dV) {
    case 8: return run_backward<DK, 8, T>(q, k, v, dout, dq, dk, dv, BH, N, P, s);
    case 16: return run_backward<DK, 16, T>(q, k, v, dout, dq, dk, dv, BH, N, P, s);
    case 32: return run_backward<DK, 32, T>(q, k, v, dout, dq, dk, dv, BH, N, P, s);
    case 64: return run_backward<DK, 64, T>(q, k, v, dout, dq, dk, dv, BH, N, P, s);
  }
  return SATA_ERR_UNSUPPORTED;
}

template <typename T>
int dispatch_dk(int dK, int dV, const void *q, const void *k, const void *v, const float *dout,
                float *dq, float *dk, float *dv, int BH, int N, int P, cudaStream_t s) {
  switch (dK) {
    case 8: return dispatch_dv<8, T>(dV, q, k, v, dout, dq, dk, dv, BH, N, P, s);
    case 16: return dispatch_dv<16, T>(dV, q, k, v, dout, dq, dk, dv, BH, N, P, s);
    case 32: return dispatch_dv<32, T>(dV, q, k, v, dout, dq, dk, dv, BH, N, P, s);
    case 64: return dispatch_dv<64, T>(dV, q, k, v, dout, dq, dk, dv, BH, N, P, s);
  }
  return SATA_ERR_UNSUPPORTED;
}

}  // namespace

int launch_backward(const void *q, const void *k, const void *v, const float *dout, float *dq,
                    float *dk, float *dv, int B, int H, int N, int dK, int dV, int P, bool bf16,
                    cudaStream_t stream) {
  const int BH = B * H;
  if (bf16)
    return dispatch_dk<__nv_bfloat16>(dK, dV, q, k, v, dout, dq, dk, dv, BH, N, P, stream);
  return dispatch_dk<float>(dK, dV, q, k, v, dout, dq, dk, dv, BH, N, P, stream);
}

}  // namespace sata
