// fp32 CUDA-core prefill for causal SATA attention (any supported dK, dV, P).
//
// Decomposition (chunked form of the per-token procedure of
// "对称性感知泰勒近似注意力机制的恒定计算成本工程实现", section
// "恒定计算成本的工程实现"): the sequence is cut into chunks of C tokens.
//   kernel 1 (chunk states): for a tile of basis rows, runs the state update
//     S += phi(k_t) [v_t, 1]^T over all tokens in order and stores S at every
//     chunk boundary (the state before chunk c) plus the final state.
//   kernel 2 (readout): for a block of tokens in chunk c,
//     [num, den]_i = phi(q_i)^T S_(before c)  +  sum_{c0 <= j <= i} T_P(s_ij) [v_j, 1]
//     and out_i = num_i / den_i.
// A continued prefill starts kernel 1 from the caller's state S_0 instead of
// zero and stores S_0 as the state before chunk 0 (snapshot slot 0); the
// snapshot before chunk c then sits in slot c instead of c - 1.
// Both terms are exact reorganisations of sum_{j<=i} T_P(s_ij)[v_j,1]
// ("对称张量分解的核心洞察": phi(q).phi(k) = T_P(q.k/sqrt(dK)) over the minimal
// basis), so the result equals the quadratic form up to rounding.
#include <algorithm>

#include "common.cuh"
#include "sata_internal.h"

namespace sata {
namespace {

constexpr int kThreads = 256;
constexpr int kFT = 32;  // basis rows per tile
constexpr int kTT = 32;  // tokens per step
constexpr int kTB = 32;  // query tokens per readout block

// Register tile of a thread: 4 consecutive rows (basis rows, or tokens in the
// readout) starting at 4 * (tid / 32) by the columns tid % 32 + 32 j < D1.
// Per reduction step it reads its 4 row values with one broadcast 16-byte
// shared load and one value per column, for 4 FMAs per column.
constexpr int kRowsT = 4;
static_assert(kThreads / 32 * kRowsT == kFT && kFT == kTT && kTT == kTB, "tile geometry");
template <int D1> struct ColTile { static constexpr int n = (D1 + 31) / 32; };

template <int DK, int DV, typename T>
__global__ void __launch_bounds__(kThreads)
    simt_chunk_states(const T *__restrict__ k, const T *__restrict__ v,
                      const uint32_t *__restrict__ idx, const float *__restrict__ w,
                      int m, int N, int C, int head0, float *__restrict__ snap, int nsnap,
                      int cont, float *__restrict__ state) {
  constexpr int D1 = DV + 1;
  constexpr int RC = ColTile<D1>::n;
  __shared__ float ks[kTT][DK + 1];
  __shared__ float vs[kTT][D1];
  __shared__ __align__(16) float ph[kTT][kFT];  // ph[t][a]: row a of token t
  __shared__ uint32_t sidx[kFT];
  __shared__ float sw[kFT];

  const int tid = threadIdx.x;
  const int ty = tid >> 5, tx = tid & 31;
  const int a0 = blockIdx.x * kFT;
  const size_t bh = (size_t)head0 + blockIdx.y;
  if (tid < kFT) {
    const int a = a0 + tid;
    sidx[tid] = a < m ? idx[a] : padding_row(DK);
    sw[tid] = a < m ? w[a] : 0.f;
  }
  float acc[kRowsT][RC];
  float *st = state + bh * (size_t)m * D1;
  // entry (row a0 + 4 ty + i, column tx + 32 j) of the tile, if it exists
  auto live = [&](int i, int j) { return a0 + kRowsT * ty + i < m && tx + 32 * j < D1; };
  auto at = [&](int i, int j) { return (size_t)(a0 + kRowsT * ty + i) * D1 + tx + 32 * j; };
#pragma unroll
  for (int i = 0; i < kRowsT; ++i)
#pragma unroll
    for (int j = 0; j < RC; ++j)
      // a continued prefill starts from the caller's state (read here, by the
      // thread that overwrites the same entries at the end)
      acc[i][j] = (cont && live(i, j)) ? st[at(i, j)] : 0.f;
  const T *kh = k + bh * N * DK;
  const T *vh = v + bh * N * DV;

  for (int t0 = 0; t0 < N; t0 += kTT) {
    if ((t0 > 0 || cont) && t0 % C == 0) {
      float *sp = snap + ((size_t)blockIdx.y * nsnap + (t0 / C - 1 + cont)) * (size_t)m * D1;
#pragma unroll
      for (int i = 0; i < kRowsT; ++i)
#pragma unroll
        for (int j = 0; j < RC; ++j)
          if (live(i, j)) sp[at(i, j)] = acc[i][j];
    }
    __syncthreads();
    for (int e = tid; e < kTT * (DK + 1); e += kThreads) {
      const int t = e / (DK + 1), i = e % (DK + 1);
      float x = 1.f;
      if (i < DK) x = (t0 + t < N) ? to_f32(kh[(size_t)(t0 + t) * DK + i]) : 0.f;
      ks[t][i] = x;
    }
    for (int e = tid; e < kTT * D1; e += kThreads) {
      const int t = e / D1, c = e % D1;
      float x = 0.f;
      if (t0 + t < N) x = (c < DV) ? to_f32(vh[(size_t)(t0 + t) * DV + c]) : 1.f;
      vs[t][c] = x;
    }
    __syncthreads();
    for (int e = tid; e < kTT * kFT; e += kThreads) {
      const int t = e / kFT, a = e % kFT;
      ph[t][a] = feature_from_packed(ks[t], sidx[a], sw[a]);
    }
    __syncthreads();
#pragma unroll 4
    for (int t = 0; t < kTT; ++t) {
      const float4 f = *reinterpret_cast<const float4 *>(&ph[t][kRowsT * ty]);
      const float fr[kRowsT] = {f.x, f.y, f.z, f.w};
#pragma unroll
      for (int j = 0; j < RC; ++j) {
        const float x = (tx + 32 * j < D1) ? vs[t][tx + 32 * j] : 0.f;
#pragma unroll
        for (int i = 0; i < kRowsT; ++i) acc[i][j] = fmaf(fr[i], x, acc[i][j]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < kRowsT; ++i)
#pragma unroll
    for (int j = 0; j < RC; ++j)
      if (live(i, j)) st[at(i, j)] = acc[i][j];
}

template <int DK, int DV, typename T>
__global__ void __launch_bounds__(kThreads)
    simt_readout(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                 const uint32_t *__restrict__ idx, const float *__restrict__ w, int m, int N,
                 int C, int P, int head0, const float *__restrict__ snap, int nsnap,
                 int cont, float *__restrict__ out) {
  constexpr int D1 = DV + 1;
  constexpr int RC = ColTile<D1>::n;
  __shared__ float qs[kTB][DK + 1];
  __shared__ float ks[kTT][DK + 1];
  __shared__ float vs[kTT][D1];
  // pt[r][t]: the reduction index r (basis row, or key) outer and the token
  // contiguous, so a thread's 4 tokens are one 16-byte load
  __shared__ __align__(16) float pt[kFT][kTB];
  __shared__ float sn[kFT][D1];
  __shared__ uint32_t sidx[kFT];
  __shared__ float sw[kFT];

  const int tid = threadIdx.x;
  const int ty = tid >> 5, tx = tid & 31;
  const int t0 = blockIdx.x * kTB;
  const size_t bh = (size_t)head0 + blockIdx.y;
  const int chunk = t0 / C;
  const int c0 = chunk * C;
  const T *qh = q + bh * N * DK;
  const T *kh = k + bh * N * DK;
  const T *vh = v + bh * N * DV;

  for (int e = tid; e < kTB * (DK + 1); e += kThreads) {
    const int t = e / (DK + 1), i = e % (DK + 1);
    float x = 1.f;
    if (i < DK) x = (t0 + t < N) ? to_f32(qh[(size_t)(t0 + t) * DK + i]) : 0.f;
    qs[t][i] = x;
  }
  float acc[kRowsT][RC];
#pragma unroll
  for (int i = 0; i < kRowsT; ++i)
#pragma unroll
    for (int j = 0; j < RC; ++j) acc[i][j] = 0.f;
  // acc[i][j] += sum_r pt[r][4 ty + i] * b[r][tx + 32 j] over kFT reduction rows
  auto accumulate = [&](const float (*b)[D1]) {
#pragma unroll 4
    for (int r = 0; r < kFT; ++r) {
      const float4 f = *reinterpret_cast<const float4 *>(&pt[r][kRowsT * ty]);
      const float fr[kRowsT] = {f.x, f.y, f.z, f.w};
#pragma unroll
      for (int j = 0; j < RC; ++j) {
        const float x = (tx + 32 * j < D1) ? b[r][tx + 32 * j] : 0.f;
#pragma unroll
        for (int i = 0; i < kRowsT; ++i) acc[i][j] = fmaf(fr[i], x, acc[i][j]);
      }
    }
  };

  // inter-chunk: phi(q_i)^T S_(before chunk)
  if (chunk > 0 || cont) {
    const float *sp = snap + ((size_t)blockIdx.y * nsnap + (chunk - 1 + cont)) * (size_t)m * D1;
    for (int a0 = 0; a0 < m; a0 += kFT) {
      __syncthreads();
      if (tid < kFT) {
        const int a = a0 + tid;
        sidx[tid] = a < m ? idx[a] : padding_row(DK);
        sw[tid] = a < m ? w[a] : 0.f;
      }
      for (int e = tid; e < kFT * D1; e += kThreads) {
        const int a = e / D1, c = e % D1;
        sn[a][c] = (a0 + a < m) ? sp[(size_t)(a0 + a) * D1 + c] : 0.f;
      }
      __syncthreads();
      for (int e = tid; e < kTB * kFT; e += kThreads) {
        const int t = e % kTB, a = e / kTB;
        pt[a][t] = feature_from_packed(qs[t], sidx[a], sw[a]);
      }
      __syncthreads();
      accumulate(sn);
    }
  }

  // intra-chunk: sum_{c0 <= j <= i} T_P(s_ij) [v_j, 1]
  const float scale = 1.0f / sqrtf((float)DK);
  const int jend = min(t0 + kTB, N);
  for (int j0 = c0; j0 < jend; j0 += kTT) {
    __syncthreads();
    for (int e = tid; e < kTT * (DK + 1); e += kThreads) {
      const int j = e / (DK + 1), i = e % (DK + 1);
      float x = 0.f;
      if (i < DK && j0 + j < jend) x = to_f32(kh[(size_t)(j0 + j) * DK + i]);
      ks[j][i] = x;
    }
    for (int e = tid; e < kTT * D1; e += kThreads) {
      const int j = e / D1, c = e % D1;
      float x = 0.f;
      if (j0 + j < jend) x = (c < DV) ? to_f32(vh[(size_t)(j0 + j) * DV + c]) : 1.f;
      vs[j][c] = x;
    }
    __syncthreads();
    for (int e = tid; e < kTB * kTT; e += kThreads) {
      const int t = e % kTB, j = e / kTB;
      float s = 0.f;
#pragma unroll
      for (int i = 0; i < DK; ++i) s = fmaf(qs[t][i], ks[j][i], s);
      const bool keep = (j0 + j <= t0 + t) && (j0 + j < jend);
      pt[j][t] = keep ? taylor_trunc(s * scale, P) : 0.f;
    }
    __syncthreads();
    accumulate(vs);
  }

  // normalise
  __syncthreads();
#pragma unroll
  for (int i = 0; i < kRowsT; ++i)
#pragma unroll
    for (int j = 0; j < RC; ++j)
      if (tx + 32 * j < D1) sn[kRowsT * ty + i][tx + 32 * j] = acc[i][j];
  __syncthreads();
  for (int e = tid; e < kTB * DV; e += kThreads) {
    const int t = e / DV, c = e % DV;
    if (t0 + t < N) out[(bh * N + t0 + t) * DV + c] = sn[t][c] / sn[t][DV];
  }
}

template <int DK, int DV, typename T>
int run_simt(const void *q, const void *k, const void *v, float *out, float *state, int BH,
             int N, int P, bool cont, const DeviceBasis *basis, cudaStream_t stream) {
  const int m = (int)basis->m;
  constexpr int D1 = DV + 1;
  // Chunk length: a multiple of 64 giving at most 16 chunks.
  const int C = std::max(64, ((N + 16 * 64 - 1) / (16 * 64)) * 64);
  const int nchunks = (N + C - 1) / C;
  const int nsnap = nchunks - 1 + (cont ? 1 : 0);  // + slot 0 = initial state
  const size_t per_head = (size_t)std::max(nsnap, 0) * m * D1 * sizeof(float);
  const size_t budget = (size_t)1 << 30;
  int G = BH;
  if (per_head > 0) G = (int)std::max<size_t>(1, std::min<size_t>(BH, budget / per_head));
  float *snap = nullptr;
  if (per_head > 0) {
    int st = SATA_OK;
    snap = (float *)get_workspace(stream, per_head * G, &st);
    if (!snap) return st;
  }
  const T *qq = (const T *)q, *kk = (const T *)k, *vv = (const T *)v;
  for (int h0 = 0; h0 < BH; h0 += G) {
    const int g = std::min(G, BH - h0);
    dim3 g1((m + kFT - 1) / kFT, g);
    prof_kernel_begin(stream, K_SIMT_CHUNK_STATES);
    simt_chunk_states<DK, DV, T><<<g1, kThreads, 0, stream>>>(kk, vv, basis->idx, basis->w, m, N,
                                                               C, h0, snap, nsnap, cont ? 1 : 0,
                                                               state);
    prof_kernel_end(stream);
    dim3 g2((N + kTB - 1) / kTB, g);
    prof_kernel_begin(stream, K_SIMT_READOUT);
    simt_readout<DK, DV, T><<<g2, kThreads, 0, stream>>>(qq, kk, vv, basis->idx, basis->w, m, N,
                                                          C, P, h0, snap, nsnap, cont ? 1 : 0,
                                                          out);
    prof_kernel_end(stream);
  }
  return cuda_status(cudaGetLastError());
}

template <typename T>
int dispatch_dv(int dK, int dV, const void *q, const void *k, const void *v, float *out,
                float *state, int BH, int N, int P, bool cont, const DeviceBasis *b,
                cudaStream_t s) {
#define SATA_CASE(DKV, DVV)        \
  if (dK == DKV && dV == DVV)      \
    return run_simt<DKV, DVV, T>(q, k, v, out, state, BH, N, P, cont, b, s);
#define SATA_ROW(DKV) SATA_CASE(DKV, 8) SATA_CASE(DKV, 16) SATA_CASE(DKV, 32) SATA_CASE(DKV, 64)
  SATA_ROW(8) SATA_ROW(16) SATA_ROW(32) SATA_ROW(64)
#undef SATA_ROW
#undef SATA_CASE
  return SATA_ERR_UNSUPPORTED;
}

}  // namespace

int launch_prefill_simt(const void *q, const void *k, const void *v, float *out, float *state,
                        int B, int H, int N, int dK, int dV, int P, bool bf16, bool cont,
                        const DeviceBasis *basis, cudaStream_t stream) {
  const int BH = B * H;
  if (bf16)
    return dispatch_dv<__nv_bfloat16>(dK, dV, q, k, v, out, state, BH, N, P, cont, basis,
                                      stream);
  return dispatch_dv<float>(dK, dV, q, k, v, out, state, BH, N, P, cont, basis, stream);
}

}  // namespace sata
