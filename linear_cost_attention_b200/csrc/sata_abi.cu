// C ABI of the SATA attention library: argument validation, per-device caches
// (basis tables, scratch workspace, device error word) and kernel dispatch.
// Declarations and the contract of every entry point are in include/sata.h.
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>
#include <vector>

#include "sata_internal.h"
#include "tc_common.cuh"
#include "tile_order.h"

namespace sata {
namespace {

struct DeviceCache {
  std::map<std::pair<int, int>, DeviceBasis *> bases;
  std::map<cudaStream_t, std::pair<void *, size_t>> workspaces;
  int *err = nullptr;  // device error word
};

// Guards the caches and the profiling records, and is held for the whole of
// every prefill / decode call (recursive: the call's helpers lock it again).
std::recursive_mutex g_mutex;
std::map<int, DeviceCache> g_devices;

DeviceCache &cache_for_current_device(int *dev_out) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev_out) *dev_out = dev;
  return g_devices[dev];
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
  const uintptr_t a0 = (uintptr_t)a, b0 = (uintptr_t)b;
  return a0 < b0 + nb && b0 < a0 + na;
}

bool supported_dim(int d) { return d == 8 || d == 16 || d == 32 || d == 64; }

void free_basis(DeviceBasis *b) {
  if (!b) return;
  cudaFree(b->idx);
  cudaFree(b->w);
  cudaFree(b->tile_desc);
  cudaFree(b->grp_idx);
  cudaFree(b->grp_slot);
  cudaFree(b->grp_row);
  cudaFree(b->grp_w);
  delete b;
}

}  // namespace

const DeviceBasis *get_device_basis(int dK, int P, int *status) {
  std::lock_guard<std::recursive_mutex> lock(g_mutex);
  DeviceCache &dc = cache_for_current_device(nullptr);
  auto it = dc.bases.find({dK, P});
  if (it != dc.bases.end()) return it->second;
  HostBasis hb = build_host_basis(dK, P);
  std::vector<uint32_t> idx(hb.m);
  std::vector<float> w(hb.m);
  for (int64_t r = 0; r < hb.m; ++r) {
    idx[r] = pack_row(hb, r);
    w[r] = (float)hb.weight[r];
  }
  DeviceBasis *db = new DeviceBasis();
  db->dK = dK;
  db->P = P;
  db->m = hb.m;
  bool ok = cudaMalloc(&db->idx, hb.m * sizeof(uint32_t)) == cudaSuccess &&
            cudaMalloc(&db->w, hb.m * sizeof(float)) == cudaSuccess &&
            cudaMemcpy(db->idx, idx.data(), hb.m * sizeof(uint32_t), cudaMemcpyHostToDevice) ==
                cudaSuccess &&
            cudaMemcpy(db->w, w.data(), hb.m * sizeof(float), cudaMemcpyHostToDevice) ==
                cudaSuccess;
  if (ok && (dK == 64 || dK == 32) && P == 4) {
    // tile order for the tensor-core path, padded to an even number of tiles
    TileOrder to;
    if (!build_tile_order(dK, &to)) {
      free_basis(db);
      *status = SATA_ERR_CUDA;
      return nullptr;
    }
    if (to.n_tiles % 2) {
      to.tiles.push_back({T_PAD, 0, 0, 0, 0, 0, 0, 0});
      to.row_of_slot.insert(to.row_of_slot.end(), 64, -1);
      to.n_tiles++;
    }
    db->n_tiles = to.n_tiles;
    db->m_pad = (int64_t)to.n_tiles * 64;
    // row groups of the state kernel (their slots index the padded tile order)
    StateGroups sg;
    if (!build_state_groups(dK, to, &sg)) {
      free_basis(db);
      *status = SATA_ERR_CUDA;
      return nullptr;
    }
    db->n_grp = sg.n_items;
    auto upload = [&](auto **dst, const auto &vec) {
      const size_t bytes = vec.size() * sizeof(vec[0]);
      return cudaMalloc((void **)dst, bytes) == cudaSuccess &&
             cudaMemcpy(*dst, vec.data(), bytes, cudaMemcpyHostToDevice) == cudaSuccess;
    };
    ok = upload(&db->grp_idx, sg.lane_idx) && upload(&db->grp_slot, sg.slot) &&
         upload(&db->grp_row, sg.row) && upload(&db->grp_w, sg.weight) &&
         cudaMalloc(&db->tile_desc, to.tiles.size() * sizeof(TileDesc)) == cudaSuccess &&
         cudaMemcpy(db->tile_desc, to.tiles.data(), to.tiles.size() * sizeof(TileDesc),
                    cudaMemcpyHostToDevice) == cudaSuccess;
  }
  // cudaMemcpy from pageable memory may return before the DMA has landed, and
  // kernels on a non-blocking stream are not ordered after the legacy stream:
  // finish the copies before any launch can read the tables.
  if (ok && cudaDeviceSynchronize() != cudaSuccess) ok = false;
  if (!ok) {
    cudaGetLastError();
    free_basis(db);
    *status = SATA_ERR_NOMEM;
    return nullptr;
  }
  dc.bases[{dK, P}] = db;
  return db;
}

void *get_workspace(cudaStream_t stream, size_t bytes, int *status) {
  std::lock_guard<std::recursive_mutex> lock(g_mutex);
  DeviceCache &dc = cache_for_current_device(nullptr);
  auto &ws = dc.workspaces[stream];
  if (ws.second >= bytes && ws.first) return ws.first;
  if (ws.first) {
    // the previous buffer may still be read by work queued on this stream
    cudaStreamSynchronize(stream);
    cudaFree(ws.first);
    ws.first = nullptr;
    ws.second = 0;
  }
  size_t sz = bytes + (bytes >> 3);  // some headroom for growth
  sz = (sz + 255) & ~(size_t)255;
  if (cudaMalloc(&ws.first, sz) != cudaSuccess) {
    cudaGetLastError();
    ws.first = nullptr;
    *status = SATA_ERR_NOMEM;
    return nullptr;
  }
  ws.second = sz;
  return ws.first;
}

int *device_error_ptr() {
  std::lock_guard<std::recursive_mutex> lock(g_mutex);
  DeviceCache &dc = cache_for_current_device(nullptr);
  if (!dc.err) {
    if (cudaMalloc(&dc.err, sizeof(int)) != cudaSuccess) {
      cudaGetLastError();
      dc.err = nullptr;
      return nullptr;
    }
    // zeroed before any kernel (on any stream) can record into it
    if (cudaMemset(dc.err, 0, sizeof(int)) != cudaSuccess ||
        cudaDeviceSynchronize() != cudaSuccess) {
      cudaGetLastError();
      cudaFree(dc.err);
      dc.err = nullptr;
      return nullptr;
    }
  }
  return dc.err;
}

int read_and_clear_device_error() {
  int *p = device_error_ptr();
  if (!p) return 0;
  int h = 0;
  if (cudaMemcpy(&h, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return -1;
  if (h && (cudaMemset(p, 0, sizeof(int)) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess))
    return -1;
  return h;
}

// ---------------------------------------------------------------- profiling
namespace {
struct ProfRec {
  int id;
  cudaEvent_t a, b;
};
bool g_prof_on = false;
std::vector<ProfRec> g_prof;       // records of the most recent call
std::vector<cudaEvent_t> g_events;  // pool, reused
size_t g_next_event = 0;

cudaEvent_t prof_event() {
  if (g_next_event == g_events.size()) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    g_events.push_back(e);
  }
  return g_events[g_next_event++];
}
}  // namespace

void prof_call_begin() {
  std::lock_guard<std::recursive_mutex> lock(g_mutex);
  if (!g_prof_on) return;
  g_prof.clear();
  g_next_event = 0;
}

void prof_kernel_begin(cudaStream_t s, int id) {
  std::lock_guard<std::recursive_mutex> lock(g_mutex);
  if (!g_prof_on) return;
  ProfRec r{id, prof_event(), prof_event()};
  if (r.a) cudaEventRecord(r.a, s);
  g_prof.push_back(r);
}

void prof_kernel_end(cudaStream_t s) {
  std::lock_guard<std::recursive_mutex> lock(g_mutex);
  if (!g_prof_on || g_prof.empty()) return;
  if (g_prof.back().b) cudaEventRecord(g_prof.back().b, s);
}

}  // namespace sata

using namespace sata;

extern "C" int sata_profile_enable(int on) {
  std::lock_guard<std::recursive_mutex> lock(g_mutex);
  const int prev = g_prof_on ? 1 : 0;
  g_prof_on = on != 0;
  return prev;
}

extern "C" int sata_profile_read(float *ms_out, int *ids_out, int cap) {
  std::lock_guard<std::recursive_mutex> lock(g_mutex);
  const int n = (int)g_prof.size();
  for (int i = 0; i < n && i < cap; ++i) {
    float ms = 0.f;
    if (!g_prof[i].a || !g_prof[i].b) return -1;
    if (cudaEventSynchronize(g_prof[i].b) != cudaSuccess) return -1;
    if (cudaEventElapsedTime(&ms, g_prof[i].a, g_prof[i].b) != cudaSuccess) return -1;
    if (ms_out) ms_out[i] = ms;
    if (ids_out) ids_out[i] = g_prof[i].id;
  }
  return n;
}

extern "C" const char *sata_kernel_name(int id) {
  switch (id) {
    case K_SIMT_CHUNK_STATES: return "simt_chunk_states";
    case K_SIMT_READOUT: return "simt_readout";
    case K_DECODE_STREAM: return "decode_stream";
    case K_DECODE_FINALIZE: return "decode_finalize";
    case K_TC_CHUNK_STATES: return "tc_chunk_states";
    case K_TC_READOUT: return "tc_readout";
    case K_TC_PREP: return "tc_prep";
    case K_DECODE_BULK: return "decode_bulk";
    case K_BWD_ROWS: return "bwd_rows";
    case K_BWD_COLS: return "bwd_cols";
  }
  return "unknown";
}

namespace {

// sata_prefill (cont = false) and sata_prefill_continue (cont = true).
int prefill_impl(const void *q, const void *k, const void *v, float *out, float *state, int B,
                 int H, int N, int dK, int dV, int P, sata_dtype dt, sata_stream_t stream,
                 bool cont) {
  if (!q || !k || !v || !out || !state) return SATA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(state))
    return SATA_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 1) return SATA_ERR_INVALID_ARG;
  if (dt != SATA_F32 && dt != SATA_BF16) return SATA_ERR_INVALID_ARG;
  if (!supported_dim(dK) || !supported_dim(dV) || P < 1 || P > kMaxP) return SATA_ERR_UNSUPPORTED;
  const long long BHN = (long long)B * H * N;
  if (BHN * (dK > dV ? dK : dV) >= (1LL << 31)) return SATA_ERR_INVALID_ARG;
  const int64_t m = count_basis(dK, P);
  const size_t es = dt == SATA_F32 ? 4 : 2;
  const size_t nq = BHN * dK * es, nv = BHN * dV * es, no = BHN * dV * 4;
  const size_t ns = (size_t)B * H * m * (dV + 1) * 4;
  if (overlaps(out, no, q, nq) || overlaps(out, no, k, nq) || overlaps(out, no, v, nv) ||
      overlaps(state, ns, q, nq) || overlaps(state, ns, k, nq) || overlaps(state, ns, v, nv) ||
      overlaps(out, no, state, ns))
    return SATA_ERR_INVALID_ARG;
  std::lock_guard<std::recursive_mutex> lock(g_mutex);  // one call at a time
  int st = SATA_OK;
  const DeviceBasis *basis = get_device_basis(dK, P, &st);
  if (!basis) return st;
  prof_call_begin();
  const bool bf16 = dt == SATA_BF16;
  static const bool force_simt = getenv("SATA_FORCE_SIMT") && getenv("SATA_FORCE_SIMT")[0] == '1';
  if (!force_simt && tc_supported(dK, dV, P, bf16) && basis->tile_desc) {
    int *err = device_error_ptr();
    if (!err) return SATA_ERR_NOMEM;
    return launch_prefill_tc(q, k, v, out, state, B, H, N, cont, basis, err,
                             (cudaStream_t)stream);
  }
  return launch_prefill_simt(q, k, v, out, state, B, H, N, dK, dV, P, bf16, cont, basis,
                             (cudaStream_t)stream);
}

}  // namespace

extern "C" int sata_prefill(const void *q, const void *k, const void *v, float *out,
                            float *state, int B, int H, int N, int dK, int dV, int P,
                            sata_dtype dt, sata_stream_t stream) {
  return prefill_impl(q, k, v, out, state, B, H, N, dK, dV, P, dt, stream, false);
}

extern "C" int sata_prefill_continue(const void *q, const void *k, const void *v, float *out,
                                     float *state, int B, int H, int N, int dK, int dV, int P,
                                     sata_dtype dt, sata_stream_t stream) {
  return prefill_impl(q, k, v, out, state, B, H, N, dK, dV, P, dt, stream, true);
}

extern "C" int sata_decode_step(const void *q, const void *k, const void *v, float *state,
                                float *out, int B, int H, int dK, int dV, int P, sata_dtype dt,
                                sata_stream_t stream) {
  if (!q || !k || !v || !out || !state) return SATA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(state))
    return SATA_ERR_INVALID_ARG;
  if (B < 1 || H < 1) return SATA_ERR_INVALID_ARG;
  if (dt != SATA_F32 && dt != SATA_BF16) return SATA_ERR_INVALID_ARG;
  if (!supported_dim(dK) || !supported_dim(dV) || P < 1 || P > kMaxP) return SATA_ERR_UNSUPPORTED;
  const long long BH = (long long)B * H;
  const int64_t m = count_basis(dK, P);
  if (BH * m * (dV + 1) >= (1LL << 40)) return SATA_ERR_INVALID_ARG;
  // head and output indices are 32-bit in the kernels
  if (BH * (dK > dV + 1 ? dK : dV + 1) >= (1LL << 31)) return SATA_ERR_INVALID_ARG;
  const size_t es = dt == SATA_F32 ? 4 : 2;
  const size_t nq = BH * dK * es, nv = BH * dV * es, no = BH * dV * 4;
  const size_t ns = (size_t)BH * m * (dV + 1) * 4;
  if (overlaps(out, no, q, nq) || overlaps(out, no, k, nq) || overlaps(out, no, v, nv) ||
      overlaps(state, ns, q, nq) || overlaps(state, ns, k, nq) || overlaps(state, ns, v, nv) ||
      overlaps(out, no, state, ns))
    return SATA_ERR_INVALID_ARG;
  std::lock_guard<std::recursive_mutex> lock(g_mutex);  // one call at a time
  int st = SATA_OK;
  const DeviceBasis *basis = get_device_basis(dK, P, &st);
  if (!basis) return st;
  prof_call_begin();
  if (bulk_decode_supported(dV))
    return launch_decode_bulk(q, k, v, state, nullptr, B, H, dK, dV, (int)m, 0, dt == SATA_BF16,
                              basis, out, (cudaStream_t)stream);
  return launch_decode(q, k, v, state, out, B, H, dK, dV, P, dt == SATA_BF16, basis,
                       (cudaStream_t)stream);
}

// ------------------------------------------------ mixed-precision decode state
namespace {

// Rows per head kept in fp32 in the mixed state: every row of degree <= 2.
int64_t mixed_lo_rows(int dK, int P) { return count_basis(dK, P < 3 ? P : 3); }

// Shared validation of the mixed-state calls; fills m, m_lo.
int check_mixed(const float *lo, const void *hi, int B, int H, int dK, int dV, int P,
                int64_t *m, int64_t *m_lo) {
  if (!lo || !aligned16(lo) || !aligned16(hi)) return SATA_ERR_INVALID_ARG;
  if (B < 1 || H < 1) return SATA_ERR_INVALID_ARG;
  if (!supported_dim(dK) || !supported_dim(dV) || P < 1 || P > kMaxP) return SATA_ERR_UNSUPPORTED;
  *m = count_basis(dK, P);
  *m_lo = mixed_lo_rows(dK, P);
  if (*m > *m_lo && !hi) return SATA_ERR_INVALID_ARG;
  const long long BH = (long long)B * H;
  if (BH * *m * (dV + 1) >= (1LL << 40)) return SATA_ERR_INVALID_ARG;
  if (BH * (dK > dV + 1 ? dK : dV + 1) >= (1LL << 31)) return SATA_ERR_INVALID_ARG;
  const size_t nlo = (size_t)BH * *m_lo * (dV + 1) * 4, nhi = (size_t)BH * (*m - *m_lo) * (dV + 1) * 2;
  if (hi && nhi && overlaps(lo, nlo, hi, nhi)) return SATA_ERR_INVALID_ARG;
  return SATA_OK;
}

}  // namespace

extern "C" int64_t sata_state_fp32_rows(int dK, int P) {
  if (dK < 1 || P < 1) return -1;
  return mixed_lo_rows(dK, P);
}

extern "C" int sata_state_split(const float *state, float *state_lo, void *state_hi, int B, int H,
                                int dK, int dV, int P, sata_stream_t stream) {
  int64_t m = 0, m_lo = 0;
  if (!state || !aligned16(state)) return SATA_ERR_INVALID_ARG;
  const int st = check_mixed(state_lo, state_hi, B, H, dK, dV, P, &m, &m_lo);
  if (st != SATA_OK) return st;
  const long long BH = (long long)B * H;
  const size_t ns = (size_t)BH * m * (dV + 1) * 4, nlo = (size_t)BH * m_lo * (dV + 1) * 4,
               nhi = (size_t)BH * (m - m_lo) * (dV + 1) * 2;
  if (overlaps(state, ns, state_lo, nlo) || (nhi && overlaps(state, ns, state_hi, nhi)))
    return SATA_ERR_INVALID_ARG;
  std::lock_guard<std::recursive_mutex> lock(g_mutex);
  return launch_state_convert(true, const_cast<float *>(state), state_lo, state_hi, BH, (int)m,
                              (int)m_lo, dV + 1, (cudaStream_t)stream);
}

extern "C" int sata_state_join(const float *state_lo, const void *state_hi, float *state, int B,
                               int H, int dK, int dV, int P, sata_stream_t stream) {
  int64_t m = 0, m_lo = 0;
  if (!state || !aligned16(state)) return SATA_ERR_INVALID_ARG;
  const int st = check_mixed(state_lo, state_hi, B, H, dK, dV, P, &m, &m_lo);
  if (st != SATA_OK) return st;
  const long long BH = (long long)B * H;
  const size_t ns = (size_t)BH * m * (dV + 1) * 4, nlo = (size_t)BH * m_lo * (dV + 1) * 4,
               nhi = (size_t)BH * (m - m_lo) * (dV + 1) * 2;
  if (overlaps(state, ns, state_lo, nlo) || (nhi && overlaps(state, ns, state_hi, nhi)))
    return SATA_ERR_INVALID_ARG;
  std::lock_guard<std::recursive_mutex> lock(g_mutex);
  return launch_state_convert(false, state, const_cast<float *>(state_lo),
                              const_cast<void *>(state_hi), BH, (int)m, (int)m_lo, dV + 1,
                              (cudaStream_t)stream);
}

extern "C" int sata_decode_step_mixed(const void *q, const void *k, const void *v, float *state_lo,
                                      void *state_hi, float *out, int B, int H, int dK, int dV,
                                      int P, sata_dtype dt, sata_stream_t stream) {
  if (!q || !k || !v || !out) return SATA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return SATA_ERR_INVALID_ARG;
  if (dt != SATA_F32 && dt != SATA_BF16) return SATA_ERR_INVALID_ARG;
  int64_t m = 0, m_lo = 0;
  const int st0 = check_mixed(state_lo, state_hi, B, H, dK, dV, P, &m, &m_lo);
  if (st0 != SATA_OK) return st0;
  if (!bulk_decode_supported(dV)) return SATA_ERR_UNSUPPORTED;
  const long long BH = (long long)B * H;
  const size_t es = dt == SATA_F32 ? 4 : 2;
  const size_t nq = BH * dK * es, nv = BH * dV * es, no = BH * dV * 4;
  const size_t nlo = (size_t)BH * m_lo * (dV + 1) * 4, nhi = (size_t)BH * (m - m_lo) * (dV + 1) * 2;
  const void *ins[3] = {q, k, v};
  const size_t nin[3] = {nq, nq, nv};
  for (int i = 0; i < 3; ++i)
    if (overlaps(out, no, ins[i], nin[i]) || overlaps(state_lo, nlo, ins[i], nin[i]) ||
        (nhi && overlaps(state_hi, nhi, ins[i], nin[i])))
      return SATA_ERR_INVALID_ARG;
  if (overlaps(out, no, state_lo, nlo) || (nhi && overlaps(out, no, state_hi, nhi)))
    return SATA_ERR_INVALID_ARG;
  std::lock_guard<std::recursive_mutex> lock(g_mutex);  // one call at a time
  int st = SATA_OK;
  const DeviceBasis *basis = get_device_basis(dK, P, &st);
  if (!basis) return st;
  prof_call_begin();
  return launch_decode_bulk(q, k, v, state_lo, m > m_lo ? state_hi : nullptr, B, H, dK, dV,
                            (int)m_lo, (int)(m - m_lo), dt == SATA_BF16, basis, out,
                            (cudaStream_t)stream);
}

extern "C" int sata_attention_backward(const void *q, const void *k, const void *v,
                                       const float *dout, float *dq, float *dk, float *dv, int B,
                                       int H, int N, int dK, int dV, int P, sata_dtype dt,
                                       sata_stream_t stream) {
  if (!q || !k || !v || !dout || !dq || !dk || !dv) return SATA_ERR_INVALID_ARG;
  const void *ptrs[7] = {q, k, v, dout, dq, dk, dv};
  for (const void *p : ptrs)
    if (!aligned16(p)) return SATA_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 1) return SATA_ERR_INVALID_ARG;
  if (dt != SATA_F32 && dt != SATA_BF16) return SATA_ERR_INVALID_ARG;
  if (!supported_dim(dK) || !supported_dim(dV) || P < 1 || P > kMaxP) return SATA_ERR_UNSUPPORTED;
  const long long BHN = (long long)B * H * N;
  if (BHN * (dK > dV + 1 ? dK : dV + 1) >= (1LL << 31)) return SATA_ERR_INVALID_ARG;
  const size_t es = dt == SATA_F32 ? 4 : 2;
  const size_t nq = BHN * dK * es, nv = BHN * dV * es, ndq = BHN * dK * 4, ndv = BHN * dV * 4;
  const void *ins[4] = {q, k, v, dout};
  const size_t nin[4] = {nq, nq, nv, ndv};
  const void *outs[3] = {dq, dk, dv};
  const size_t nout[3] = {ndq, ndq, ndv};
  for (int o = 0; o < 3; ++o) {
    for (int i = 0; i < 4; ++i)
      if (overlaps(outs[o], nout[o], ins[i], nin[i])) return SATA_ERR_INVALID_ARG;
    for (int o2 = o + 1; o2 < 3; ++o2)
      if (overlaps(outs[o], nout[o], outs[o2], nout[o2])) return SATA_ERR_INVALID_ARG;
  }
  std::lock_guard<std::recursive_mutex> lock(g_mutex);  // one call at a time
  prof_call_begin();
  return launch_backward(q, k, v, dout, dq, dk, dv, B, H, N, dK, dV, P, dt == SATA_BF16,
                         (cudaStream_t)stream);
}

extern "C" int sata_get_error(sata_stream_t stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) {
    cudaGetLastError();
    return SATA_ERR_CUDA;
  }
  if (cudaGetLastError() != cudaSuccess) return SATA_ERR_CUDA;
  const int code = read_and_clear_device_error();
  if (code < 0) return SATA_ERR_CUDA;
  return code == 0 ? SATA_OK : SATA_ERR_TIMEOUT;
}

namespace sata {
namespace {
long long g_tc_wait_limit = 0;  // 0: the kernels' full limit
}  // namespace
long long tc_wait_limit() {
  std::lock_guard<std::recursive_mutex> lock(g_mutex);
  return g_tc_wait_limit > 0 ? g_tc_wait_limit : tc::kWaitLimitCycles;
}
}  // namespace sata

extern "C" long long sata_test_set_wait_limit(long long cycles) {
  std::lock_guard<std::recursive_mutex> lock(g_mutex);
  const long long prev = g_tc_wait_limit;
  g_tc_wait_limit = cycles > 0 ? cycles : 0;
  return prev;
}

extern "C" const char *sata_status_string(int status) {
  switch (status) {
    case SATA_OK: return "SATA_OK";
    case SATA_ERR_INVALID_ARG: return "SATA_ERR_INVALID_ARG: invalid argument";
    case SATA_ERR_UNSUPPORTED: return "SATA_ERR_UNSUPPORTED: dK, dV or P not supported";
    case SATA_ERR_CUDA: return "SATA_ERR_CUDA: a CUDA call or kernel launch failed";
    case SATA_ERR_NOMEM: return "SATA_ERR_NOMEM: device allocation failed";
    case SATA_ERR_TIMEOUT: return "SATA_ERR_TIMEOUT: a device-side wait gave up";
  }
  return "unknown sata status";
}

extern "C" void sata_release(void) {
  std::lock_guard<std::recursive_mutex> lock(g_mutex);
  int cur = 0;
  cudaGetDevice(&cur);
  for (auto &kv : g_devices) {
    cudaSetDevice(kv.first);
    for (auto &b : kv.second.bases) free_basis(b.second);
    for (auto &w : kv.second.workspaces) cudaFree(w.second.first);
    cudaFree(kv.second.err);
  }
  g_devices.clear();
  cudaSetDevice(cur);
}
