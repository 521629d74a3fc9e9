// tensor_map.cu -- host-side tensor maps for the coders' tile staging.
//
// The warp coders of tiled streams move each 4-row slice of a tile (one
// channel, the tile's width) between global and shared memory with one
// tensor-tile copy; the copy engine walks the tensor's strides, so no thread
// computes per-element addresses.  The maps are encoded with the driver's
// cuTensorMapEncodeTiled, fetched through the runtime so the library needs
// no link against the driver library.
#include <mutex>

#include <cuda.h>

#include "rans_common.cuh"
#include "rans_internal.h"

namespace rb {
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

std::mutex g_mutex;
EncodeTiledFn g_encode = nullptr;

EncodeTiledFn encode_fn() {
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_encode == nullptr) {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(f);
  }
  return g_encode;
}

}  // namespace

int encode_tile_map(void *map, const void *base, uint64_t width, uint64_t height,
                    uint64_t depth, uint32_t box_w, uint32_t box_h) {
  EncodeTiledFn f = encode_fn();
  if (f == nullptr) return RANS_ERR_CUDA;
  // 4-byte elements: the row stride and the base must be 16-byte aligned,
  // the box's row a multiple of 16 bytes
  if ((reinterpret_cast<uintptr_t>(base) & 15) != 0 || (width * 4) % 16 != 0 ||
      (box_w * 4) % 16 != 0 || box_w == 0 || box_w > 256 || box_h == 0 || box_h > 256)
    return RANS_ERR_ARG;
  const cuuint64_t dims[3] = {width, height, depth};
  const cuuint64_t strides[2] = {width * 4, width * height * 4};
  const cuuint32_t box[3] = {box_w, box_h, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = f(reinterpret_cast<CUtensorMap *>(map), CU_TENSOR_MAP_DATA_TYPE_INT32, 3,
                       const_cast<void *>(base), dims, strides, box, estr,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? RANS_OK : RANS_ERR_CUDA;
}

// Float latents on the tile kernels: tiled W = 32 streams (64-bit format,
// no alias, one scale per element) whose tiles are all 64 or 56 wide and a
// multiple of 4 rows high, the two staged tensors 16-byte aligned.
bool flt_tile_shape_ok(const Geom &g, const void *a, const void *b) {
  if (g.kind != RANS_CHUNK_TILED || g.W != 32 || g.alias || g.ib_shift != 0) return false;
  if ((reinterpret_cast<uintptr_t>(a) & 15) || (reinterpret_cast<uintptr_t>(b) & 15)) return false;
  auto width_ok = [](int64_t w) { return w == 64 || w == 56; };
  const int64_t ww1 = g.Wd % g.tw, hh1 = g.H % g.th;
  if (!width_ok(g.tw > g.Wd ? g.Wd : g.tw) || (ww1 != 0 && !width_ok(ww1))) return false;
  return g.th % 4 == 0 && hh1 % 4 == 0 && g.Wd % 4 == 0;
}

}  // namespace rb
