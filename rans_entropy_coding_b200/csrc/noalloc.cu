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
// call on each device looks the address up with cudaGetSymbolAddress (with
// that device current) and caches it; that first call should therefore come
// before any stream capture.  All calls share the array: calls whose work
// overlaps on the GPU (concurrent streams, or several host threads on one
// device) race on it and must be serialised by the caller.  Nothing here
// allocates: no cudaMalloc, no cudaFree, no allocating library routine.
#include <mutex>

#include "rans_common.cuh"
#include "rans_internal.h"

namespace {

constexpr uint64_t kStaticWorkspaceBytes = 32ull << 20;  // 32 MiB

__device__ __align__(256) unsigned char g_static_workspace[kStaticWorkspaceBytes];

std::mutex g_setup_mutex;
void *g_workspace_addr[128] = {nullptr};

// Device address of the static workspace on the current device (looked up
// once per device).
int static_workspace(void **addr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return RANS_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_workspace_addr[dev] == nullptr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess || p == nullptr)
      return RANS_ERR_CUDA;
    g_workspace_addr[dev] = p;
  }
  *addr = g_workspace_addr[dev];
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
