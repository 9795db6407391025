// sata_decode_step_noalloc: the decode step without any device allocation.
//
// Who needs it: a host that has handed all device memory to its own pool
// allocator (a framework's caching allocator that reserves the GPU), a serving
// loop that must not hit cudaMalloc/cudaFree because they can synchronise the
// device and stall other streams, or a plug-in host whose policy forbids
// allocations made behind its back.  sata_decode_step allocates lazily (basis
// tables on first use, a grow-only workspace for the per-head partial sums);
// this entry point instead keeps both in file-scope __device__ arrays that
// every GPU loading the library holds until the process exits:
//   - partial sums: kNoAllocPartials floats (256 KiB), enough for
//     B*H*(dV+1) <= 65536, e.g. B*H <= 1008 heads at dV = 64;
//   - basis tables for dK in {8, 16, 32, 64}, each built for P = 4 (rows are
//     degree-major, so the first C(dK+P-1, P-1) rows serve every P <= 4):
//     55584 rows, 434 KiB.
// The scratch is shared by every call on the device and keeps the last call's
// contents; each call clears the part it uses before its kernels run.  Calls
// whose work overlaps on the GPU (other streams, other host threads) race on
// the scratch: order them.
#include <mutex>

#include "sata_internal.h"

namespace sata {
namespace {

constexpr int kNoAllocPartials = 65536;
constexpr int kTableRows[4] = {165, 969, 6545, 47905};  // C(dK+3, 3), dK = 8, 16, 32, 64
constexpr int kTableOffset[4] = {0, 165, 165 + 969, 165 + 969 + 6545};
constexpr int kNoAllocTableRows = 165 + 969 + 6545 + 47905;

static __device__ __align__(256) float g_noalloc_partials[kNoAllocPartials];
static __device__ __align__(256) uint32_t g_noalloc_idx[kNoAllocTableRows];
static __device__ __align__(256) float g_noalloc_w[kNoAllocTableRows];

constexpr int kMaxDevices = 64;
struct NoAllocDevice {
  bool ready = false;
  float *partials = nullptr;  // device address of g_noalloc_partials
  uint32_t *idx = nullptr;    // device address of g_noalloc_idx
  float *w = nullptr;         // device address of g_noalloc_w
};
NoAllocDevice g_noalloc_dev[kMaxDevices];
std::mutex g_noalloc_mutex;

int dim_slot(int d) { return d == 8 ? 0 : d == 16 ? 1 : d == 32 ? 2 : d == 64 ? 3 : -1; }

// Once per device, with that device current: resolve the arrays' device
// addresses (in host code the array names are host-side stand-ins, not device
// addresses) and fill the tables.  Synchronous: it returns after the copies
// have landed (cudaDeviceSynchronize), so a first call made on any stream sees
// complete tables.
int noalloc_setup(int dev, NoAllocDevice **out) {
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  NoAllocDevice &d = g_noalloc_dev[dev];
  if (d.ready) {
    *out = &d;
    return SATA_OK;
  }
  if (cudaGetSymbolAddress((void **)&d.partials, g_noalloc_partials) != cudaSuccess ||
      cudaGetSymbolAddress((void **)&d.idx, g_noalloc_idx) != cudaSuccess ||
      cudaGetSymbolAddress((void **)&d.w, g_noalloc_w) != cudaSuccess) {
    cudaGetLastError();
    return SATA_ERR_CUDA;
  }
  for (int s = 0; s < 4; ++s) {
    const int dK = 8 << s;
    HostBasis hb = build_host_basis(dK, 4);
    if (hb.m != kTableRows[s]) return SATA_ERR_CUDA;
    std::vector<uint32_t> idx(hb.m);
    std::vector<float> w(hb.m);
    for (int64_t r = 0; r < hb.m; ++r) {
      idx[r] = pack_row(hb, r);
      w[r] = (float)hb.weight[r];
    }
    if (cudaMemcpy(d.idx + kTableOffset[s], idx.data(), hb.m * sizeof(uint32_t),
                   cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(d.w + kTableOffset[s], w.data(), hb.m * sizeof(float),
                   cudaMemcpyHostToDevice) != cudaSuccess) {
      cudaGetLastError();
      return SATA_ERR_CUDA;
    }
  }
  // cudaMemcpy from pageable host memory can return once the data is staged,
  // before the DMA lands, and kernels on a non-blocking stream (any
  // torch.cuda.Stream) are not ordered after the legacy stream: wait for the
  // copies before the tables can be read by any launch.
  if (cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    return SATA_ERR_CUDA;
  }
  d.ready = true;
  *out = &d;
  return SATA_OK;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
  const uintptr_t a0 = (uintptr_t)a, b0 = (uintptr_t)b;
  return a0 < b0 + nb && b0 < a0 + na;
}

}  // namespace
}  // namespace sata

extern "C" int sata_decode_step_noalloc(const void *q, const void *k, const void *v,
                                        float *state, float *out, int B, int H, int dK, int dV,
                                        int P, sata_dtype dt, sata_stream_t stream) {
  using namespace sata;
  if (!q || !k || !v || !out || !state) return SATA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(state))
    return SATA_ERR_INVALID_ARG;
  if (B < 1 || H < 1) return SATA_ERR_INVALID_ARG;
  if (dt != SATA_F32 && dt != SATA_BF16) return SATA_ERR_INVALID_ARG;
  const int slot = dim_slot(dK);
  if (slot < 0 || dim_slot(dV) < 0 || P < 1 || P > 4) return SATA_ERR_UNSUPPORTED;
  const long long BH = (long long)B * H;
  if (BH * (dV + 1) > kNoAllocPartials) return SATA_ERR_INVALID_ARG;  // scratch limit
  const int64_t m = count_basis(dK, P);
  const size_t es = dt == SATA_F32 ? 4 : 2;
  const size_t nq = BH * dK * es, nv = BH * dV * es, no = BH * dV * 4;
  const size_t ns = (size_t)BH * m * (dV + 1) * 4;
  if (overlaps(out, no, q, nq) || overlaps(out, no, k, nq) || overlaps(out, no, v, nv) ||
      overlaps(state, ns, q, nq) || overlaps(state, ns, k, nq) || overlaps(state, ns, v, nv) ||
      overlaps(out, no, state, ns))
    return SATA_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return SATA_ERR_CUDA;
  }
  NoAllocDevice *nd = nullptr;
  const int st = noalloc_setup(dev, &nd);
  if (st != SATA_OK) return st;
  return launch_decode_scratch(q, k, v, state, out, B, H, dK, dV, dt == SATA_BF16,
                               nd->idx + kTableOffset[slot], nd->w + kTableOffset[slot], m,
                               nd->partials, (cudaStream_t)stream);
}
