// Internal declarations shared by the library's translation units.
// Not part of the public ABI (see include/sata.h).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <vector>

#include "../../include/sata.h"

namespace sata {

// ------------------------------------------------------------ basis tables
// Host-side enumeration of the minimal symmetric basis (GPU path's own code).
// Row order: degree-major p = 0..P-1, lexicographic tuples i_1<=...<=i_p.
struct HostBasis {
  int dK = 0, P = 0;
  int64_t m = 0;
  std::vector<uint8_t> degree;          // [m]
  std::vector<uint8_t> ix;              // [m*4]; unused slots = dK (points at a 1.0)
  std::vector<double> weight;           // [m]  1/sqrt(alpha! * dK^(p/2))
};
HostBasis build_host_basis(int dK, int P);
int64_t count_basis(int dK, int P);  // m, or -1
constexpr int kMaxP = 5;             // degrees 0..4 (four index slots)

// Packed row for the CUDA-core kernels: four 7-bit indices (unused slots = dK,
// which points at a 1.0) and the degree in bits 28..30.
inline uint32_t pack_row(const HostBasis &hb, int64_t r) {
  uint32_t v = (uint32_t)hb.degree[r] << 28;
  for (int s = 0; s < 4; ++s) v |= (uint32_t)hb.ix[4 * r + s] << (7 * s);
  return v;
}

// Device copy of the tables in the packed form the kernels read.
//   idx[r] = i1 | i2 << 7 | i3 << 14 | i4 << 21 | degree << 28  (unused slots = dK)
//   w[r]   = fp32 weight
struct DeviceBasis {
  int dK = 0, P = 0;
  int64_t m = 0;
  uint32_t *idx = nullptr;
  float *w = nullptr;
  // Tensor-core tables (dK = 64 or 32, P == 4); null when not built.
  int n_tiles = 0;              // 64-feature tiles of the tile order (readout, snapshots)
  int64_t m_pad = 0;            // n_tiles * 64
  void *tile_desc = nullptr;    // [n_tiles] TileDesc (tile_order.h)
  int n_grp = 0;                // state-kernel items per head (StateGroups, tile_order.h)
  uint64_t *grp_idx = nullptr;  // [n_grp][128] shared and third factor rows of each lane group
  int32_t *grp_slot = nullptr;  // [n_grp][4][128] tile-order slot of each row (-1 = pad)
  int32_t *grp_row = nullptr;   // [n_grp][4][128] lexicographic row (-1 = pad)
  float *grp_w = nullptr;       // [n_grp][4][128] basis weight (0 = pad)
};

// Returns the cached tables for the current device (builds them on first use).
// Thread-safe.  Returns nullptr with *status set on failure.
const DeviceBasis *get_device_basis(int dK, int P, int *status);

// Per-(device, stream) grow-only scratch workspace.  Thread-safe.
void *get_workspace(cudaStream_t stream, size_t bytes, int *status);

// Device error word (first device-side failure code; 0 = none).
int read_and_clear_device_error();
int *device_error_ptr();

// ------------------------------------------------------------ launchers
// cont: start from the state in `state` (continued prefill) instead of zero.
int launch_prefill_simt(const void *q, const void *k, const void *v, float *out,
                        float *state, int B, int H, int N, int dK, int dV, int P,
                        bool bf16, bool cont, const DeviceBasis *basis, cudaStream_t stream);

// Tensor-core prefill (bf16, P = 4, dK = dV = 64 or 32); basis must carry the tile order.
bool tc_supported(int dK, int dV, int P, bool bf16);
// Cycles a role's wait in the tensor-core kernels may take before it gives up
// (default: the kernels' full limit; lowered only by sata_test_set_wait_limit).
long long tc_wait_limit();
int launch_prefill_tc(const void *q, const void *k, const void *v, float *out, float *state,
                      int B, int H, int N, bool cont, const DeviceBasis *basis, int *err,
                      cudaStream_t stream);

int launch_decode(const void *q, const void *k, const void *v, float *state, float *out,
                  int B, int H, int dK, int dV, int P, bool bf16,
                  const DeviceBasis *basis, cudaStream_t stream);

// Decode through shared memory with bulk async copies (dV = 32 or 64): lo holds
// the first m_lo rows of every head in fp32, hi (IEEE fp16, may be null when
// m_hi = 0) the other m_hi rows.  An fp32 state is lo with m_hi = 0.
bool bulk_decode_supported(int dV);
int launch_decode_bulk(const void *q, const void *k, const void *v, float *lo, void *hi, int B,
                       int H, int dK, int dV, int m_lo, int m_hi, bool bf16,
                       const DeviceBasis *basis, float *out, cudaStream_t stream);
// fp32 state <-> mixed state (split: state -> lo, hi; join: lo, hi -> state).
int launch_state_convert(bool split, float *state, float *lo, void *hi, long long BH, int m,
                         int m_lo, int D1, cudaStream_t stream);

// Gradients of sum(dout * out) w.r.t. q, k, v (fp32 outputs, CUDA cores).
int launch_backward(const void *q, const void *k, const void *v, const float *dout, float *dq,
                    float *dk, float *dv, int B, int H, int N, int dK, int dV, int P, bool bf16,
                    cudaStream_t stream);

// Decode with caller-supplied basis tables (packed as in DeviceBasis) and
// partial-sum scratch y of at least B*H*(dV+1) floats.
int launch_decode_scratch(const void *q, const void *k, const void *v, float *state, float *out,
                          int B, int H, int dK, int dV, bool bf16, const uint32_t *idx,
                          const float *w, int64_t m, float *y, cudaStream_t stream);

// ------------------------------------------------------------ profiling hook
enum KernelId {
  K_SIMT_CHUNK_STATES = 1,
  K_SIMT_READOUT = 2,
  K_DECODE_STREAM = 3,
  K_DECODE_FINALIZE = 4,
  K_TC_CHUNK_STATES = 5,
  K_TC_READOUT = 6,
  K_TC_PREP = 7,
  K_DECODE_BULK = 8,
  K_BWD_ROWS = 9,
  K_BWD_COLS = 10,
};
void prof_call_begin();                          // start of an entry-point call
void prof_kernel_begin(cudaStream_t s, int id);  // before a launch
void prof_kernel_end(cudaStream_t s);            // after a launch

// Status from the last CUDA call / launch.
inline int cuda_status(cudaError_t e) { return e == cudaSuccess ? SATA_OK : SATA_ERR_CUDA; }

}  // namespace sata
