// gdpa_noalloc.cu -- gdpa_forward_no_alloc: the forward for callers that
// cannot allocate device memory.
//
// Some callers have no way to hand this library a workspace: a plugin inside
// a host framework that owns every byte of device memory and offers no
// allocator hook, or a serving process that plans all of its memory at start
// and must not allocate (or ask its caller to allocate) on the request path.
// For them this entry point runs the same forward kernels with their scratch
// (the status block, the longest-first sample order, the query-tile prefix
// and the per-sample descriptors)
// in a fixed array compiled into the library.  It never calls cudaMalloc,
// cudaFree or any allocating routine.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library keeps its own copy until the process exits.  Host code cannot pass
// the array's name to a kernel (on the host it names a stand-in, not device
// memory), so the first call on each device looks up the device address with
// cudaGetSymbolAddress while that device is current and caches it; that first
// call should therefore come before any stream capture.
#include <mutex>

#include "gdpa.h"
#include "gdpa_internal.h"

namespace {

// status (256 B) + order[B] + tile_start[B+1] + info[B] (16 B each), each
// rounded up to 256 B, for the largest batch the library accepts:
// 393,728 bytes.
constexpr int kNoAllocMaxBatch = gdpa::kMaxSortBatch;
constexpr size_t kNoAllocBytes = gdpa::schedule_ws_bytes(kNoAllocMaxBatch);
static_assert(kNoAllocBytes == 393728, "documented size of the fixed scratch array");

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices];

// Device address of this device's copy of the array (looked up once per device).
void* scratch_for_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = ptr;
  }
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" GDPA_API gdpa_status_t gdpa_forward_no_alloc(
    const gdpa_params_t* p, const void* q, const void* k, const void* v,
    const int32_t* q_offsets, const int32_t* kv_offsets, const float* bias, void* o, float* lse,
    gdpa_stream_t stream) {
  if (!p) return GDPA_ERR_INVALID_ARG;
  if (p->B > kNoAllocMaxBatch) return GDPA_ERR_WORKSPACE;  // beyond the fixed scratch
  // rotary tables: Q and K are turned inside the attention kernel, which needs
  // no turned copies (and gives the same bits as the streamed turn)
  gdpa_params_t pp = *p;
  if (pp.rope_q) pp.debug_flags |= gdpa::kDebugFusedRotary;
  p = &pp;
  const size_t need = gdpa_workspace_size(p, 0);
  if (need == 0) return GDPA_ERR_INVALID_ARG;
  if (need > kNoAllocBytes) return GDPA_ERR_WORKSPACE;
  void* scratch = scratch_for_current_device();
  if (!scratch) return GDPA_ERR_CUDA;
  // The schedule kernel that starts every forward clears the status block and
  // rewrites the order and prefix in full, so nothing left by an earlier call
  // is read.
  return gdpa_forward(p, q, k, v, q_offsets, kv_offsets, bias, o, lse, scratch, kNoAllocBytes,
                      stream);
}

extern "C" GDPA_API gdpa_status_t gdpa_forward_no_alloc_status(gdpa_stream_t stream) {
  void* scratch = scratch_for_current_device();
  if (!scratch) return GDPA_ERR_CUDA;
  // the status block is the array's first 256 bytes, as in a workspace
  return gdpa_get_device_status(scratch, stream);
}
