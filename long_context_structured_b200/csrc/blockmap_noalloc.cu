// blockmap_noalloc.cu -- sattn_build_blockmap_noalloc: the block map and
// separator compaction with its scratch in a fixed device array, for callers
// that cannot give the library a workspace.
//
// Who needs this: code that runs where it may not allocate device memory or
// own a workspace buffer -- for example a plugin or callback inside a host
// framework that manages every byte of device memory itself and forbids its
// extensions from allocating, or a latency-critical loop in which an
// allocation (which can implicitly synchronise the device) is not allowed.
// Such a caller still provides the inputs and outputs; the only scratch the
// block map needs (a per-sequence prefix count of the separator flags and
// the tile-class tables derived from it) lives in the static array below.
//
// Cost and limits:
//   - every GPU that loads libsattn.so holds kNoallocScratchBytes (4 MiB)
//     for this array until the process exits;
//   - blockmap_scratch_bytes(B, T, window) must not exceed it: about
//     B * (T / 4 + T / 128 + 16 nQT min(nQT / 16, window / 2048 + 2)) bytes
//     with nQT = ceil(T / 128);
//   - all calls share the one array: calls whose executions overlap on the
//     GPU (different streams, or several host threads) race on it and give
//     undefined results; serialise them;
//   - the array keeps the previous call's contents; nothing in it has to
//     start at zero, because the scan kernel rewrites every entry the class
//     kernel reads before it reads it;
//   - the array's device address is looked up once per device and kept; a
//     cudaDeviceReset destroys the array with the context, so after a reset
//     this entry point must not be called again in the same process.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/sattn.h"
#include "kernels.cuh"
#include "prof.cuh"

namespace {

constexpr size_t kNoallocScratchBytes = size_t(1) << 22;  // 4 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_blockmap_scratch[kNoallocScratchBytes];

std::mutex g_setup_mu;
uint8_t* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  The first call
// on each device resolves it with cudaGetSymbolAddress; the name of a
// __device__ array is only a host-side stand-in, never a device pointer.
int scratch_for_current_device(uint8_t** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SATTN_ERR_CUDA;
  std::lock_guard<std::mutex> g(g_setup_mu);
  if (!g_scratch_addr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_blockmap_scratch) != cudaSuccess || !ptr) return SATTN_ERR_CUDA;
    g_scratch_addr[dev] = static_cast<uint8_t*>(ptr);
  }
  *out = g_scratch_addr[dev];
  return SATTN_OK;
}

}  // namespace

extern "C" int sattn_build_blockmap_noalloc(const sattn_params* p, const uint8_t* is_sep, uint8_t* cls,
                                            int32_t* sep_pos, int32_t* sep_count, int32_t* qtile_sep_range,
                                            void* stream) {
  if (!p || !sep_pos || !sep_count || !qtile_sep_range) return SATTN_ERR_INVALID_ARG;
  if (p->B < 1 || p->T < 1 || p->n_start < 0 || p->window < 0) return SATTN_ERR_INVALID_ARG;
  if (sattn::blockmap_scratch_bytes(p->B, p->T, p->window) > kNoallocScratchBytes) return SATTN_ERR_UNSUPPORTED;
  uint8_t* scratch = nullptr;
  int rc = scratch_for_current_device(&scratch);
  if (rc != SATTN_OK) return rc;
  sattn::BlockmapArgs a{};
  a.B = p->B;
  a.T = p->T;
  a.n_start = p->n_start;
  a.window = p->window;
  a.is_sep = is_sep;
  a.scratch = scratch;
  a.sep_pos = sep_pos;
  a.sep_count = sep_count;
  a.ranges = qtile_sep_range;
  a.cls = cls;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  sattn::ProfScope ps("blockmap_noalloc", cls ? 2 : 1, st);  // the class kernel runs only when classes are asked for
  return sattn::launch_blockmap(a, st) == cudaSuccess ? SATTN_OK : SATTN_ERR_CUDA;
}
