// noalloc.cu -- qwm_build_centroids_noalloc: the centroid build with its
// scratch in a fixed device array instead of the cache's WORKSPACE buffer.
//
// Who needs it: code that runs inside a host application which owns the GPU
// memory budget (an inference server or engine plugin host that hands its
// plugins pre-sized buffers and forbids cudaMalloc/cudaFree, which synchronize
// the device and fragment the host's pool).  Such callers can pass the cache
// buffers they were given, but cannot obtain extra scratch on demand.
//
// The scratch is a file-scope device array of QWM_NOALLOC_SCRATCH_BYTES; every
// GPU that loads this library holds it until the process exits.  Host code
// cannot use the array's name as a device address, so the address is looked up
// once per device with cudaGetSymbolAddress (with that device current) and
// cached; the first call on a device performs that lookup.
#include <mutex>

#include "common.cuh"

namespace qwm {
namespace {

__device__ __align__(256) unsigned char g_noalloc_scratch[QWM_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device (nullptr on error).
void* scratch_on_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_scratch_addr[dev] = p;
  }
  return g_scratch_addr[dev];
}

}  // namespace
}  // namespace qwm

using namespace qwm;

extern "C" qwm_status qwm_build_centroids_noalloc(qwm_cache* c, const void* K, const void* V,
                                                  int64_t n, int32_t iters, void* stream) {
  int slot = 0;
  const qwm_status st = centroid_build_slot(c, K, V, n, iters, &slot);
  if (st != QWM_OK) return st;
  Dims D = dims_of(&c->cfg);
  D.tcap = n;  // the assignment scratch holds n tokens per head, not the capacity
  const size_t need = ((size_t)D.H * D.C * D.d * 4 + 255) / 256 * 256 + (size_t)D.H * n * 4;
  if (need > (size_t)QWM_NOALLOC_SCRATCH_BYTES) return QWM_ERR_CAPACITY;
  void* scratch = scratch_on_current_device();
  if (!scratch) return QWM_ERR_CUDA;
  cudaStream_t s = (cudaStream_t)stream;
  const size_t off = (size_t)slot * cent_slot_elems(D);
  uint16_t* cent_k = (uint16_t*)c->buf.ptr[QWM_BUF_CENT_K] + off;
  uint16_t* cent_v = (uint16_t*)c->buf.ptr[QWM_BUF_CENT_V] + off;
  cudaError_t e = launch_kmeans(D, (const uint16_t*)K, n, iters, cent_k, scratch, s);
  if (e == cudaSuccess) e = launch_kmeans(D, (const uint16_t*)V, n, iters, cent_v, scratch, s);
  if (e != cudaSuccess) return QWM_ERR_CUDA;
  centroid_build_commit(c, slot);
  return QWM_OK;
}
