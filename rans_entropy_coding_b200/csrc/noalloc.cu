// noalloc.cu -- rans_encode_with_indexes_noalloc: the encoder for callers
// that cannot allocate device memory themselves.
//
// rans_encode_with_indexes needs a caller-provided workspace (a status word,
// per-stream lengths and a worst-case scratch slot per stream).  Some callers
// cannot provide one: code running inside a host framework whose allocator
// owns all device memory and must not be bypassed, or a latency-critical path
// on which cudaMalloc -- which may synchronise the whole device -- is not
// allowed.  For them this entry point uses a workspace that lives in the
// library itself: a file-scope __device__ array of kStaticWorkspaceBytes,
// which every GPU that loads the library keeps until the process exits.
//
// Host code cannot use the array's name as a device address, so the first
// call in each CUDA context looks the address up with cudaGetSymbolAddress
// (with that context's device current) and caches it beside the context's
// ID; that first call should therefore come before any stream capture.  A
// context that is destroyed and created again (a device reset) gets a new
// ID, so the next call looks the address up again instead of using the old
// one.  All calls share the array: calls whose work overlaps on the GPU
// (concurrent streams, or several host threads on one device) race on it
// and must be serialised by the caller.  Nothing here allocates: no
// cudaMalloc, no cudaFree, no allocating library routine.
#include <mutex>

#include <cuda.h>  // CUcontext / CUresult types; the entry points are fetched at run time

#include "rans_common.cuh"
#include "rans_internal.h"

namespace {

constexpr uint64_t kStaticWorkspaceBytes = 32ull << 20;  // 32 MiB

__device__ __align__(256) unsigned char g_static_workspace[kStaticWorkspaceBytes];

std::mutex g_setup_mutex;

// The context a lookup was made in, by the driver's context ID (unique for
// the life of the process, unlike a context handle, which can be reused).
struct CachedAddr {
  unsigned long long ctx_id;
  void *addr;
};
CachedAddr g_workspace_addr[128] = {};

// Driver entry points, fetched through the runtime so that the library
// needs no link against the driver library.
typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;

// ID of the context current on this thread; 0 when none is (yet) current.
// Called with g_setup_mutex held.
int current_context_id(unsigned long long *id) {
  *id = 0;
  if (g_ctx_get_current == nullptr || g_ctx_get_id == nullptr) {
    cudaDriverEntryPointQueryResult q1, q2;
    void *f1 = nullptr, *f2 = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) != cudaSuccess ||
        q1 != cudaDriverEntryPointSuccess || f1 == nullptr ||
        cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) != cudaSuccess ||
        q2 != cudaDriverEntryPointSuccess || f2 == nullptr)
      return RANS_ERR_CUDA;
    g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(f1);
    g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(f2);
  }
  CUcontext ctx = nullptr;
  if (g_ctx_get_current(&ctx) != CUDA_SUCCESS) return RANS_ERR_CUDA;
  if (ctx == nullptr) return RANS_OK;
  return g_ctx_get_id(ctx, id) == CUDA_SUCCESS ? RANS_OK : RANS_ERR_CUDA;
}

// Device address of the static workspace in the current device's context
// (looked up once per context).
int static_workspace(void **addr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return RANS_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  unsigned long long id = 0;
  int st = current_context_id(&id);
  if (st) return st;
  CachedAddr &e = g_workspace_addr[dev];
  if (id != 0 && e.addr != nullptr && e.ctx_id == id) {
    *addr = e.addr;
    return RANS_OK;
  }
  // the lookup also makes the device's context current when none was
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess || p == nullptr)
    return RANS_ERR_CUDA;
  st = current_context_id(&id);
  if (st) return st;
  if (id == 0) return RANS_ERR_CUDA;
  e.ctx_id = id;
  e.addr = p;
  *addr = p;
  return RANS_OK;
}

// Device errors from the encoder sit in the workspace's status word, which
// the caller cannot read here; mark them in the outputs instead.
__global__ void flag_error_kernel(const int32_t *status, uint64_t *stream_offsets, int64_t S) {
  if (threadIdx.x == 0 && *status != 0) stream_offsets[S] = ~0ull;
}

}  // namespace

extern "C" __attribute__((visibility("default"))) int rans_encode_with_indexes_noalloc(
    const void *symbols, int32_t sym_dtype, const int32_t *indexes, int64_t n,
    const rans_tables *tables, const rans_chunking *chunking, uint8_t *out,
    uint64_t out_capacity, uint64_t *stream_offsets, void *stream) {
  const uint64_t need = rans_encode_workspace_bytes(chunking, n);
  if (need == 0) return RANS_ERR_ARG;
  if (need > kStaticWorkspaceBytes) return RANS_ERR_CAPACITY;
  void *ws = nullptr;
  int st = static_workspace(&ws);
  if (st) return st;
  st = rans_encode_with_indexes(symbols, sym_dtype, indexes, n, tables, chunking, out,
                                out_capacity, stream_offsets, ws, kStaticWorkspaceBytes, stream);
  if (st) return st;
  const int64_t S = rans_num_streams(chunking, n);
  flag_error_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const int32_t *>(ws), stream_offsets, S);
  return cudaGetLastError() == cudaSuccess ? RANS_OK : RANS_ERR_CUDA;
}
