// api.cu -- the extern "C" entry points of librans_b200: argument checks,
// chunking geometry, workspace layout and launch order.  Every coding step
// runs in the kernels of tables.cu, encode.cu and decode.cu.
#include <cstring>
#include <mutex>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "rans_common.cuh"
#include "rans_internal.h"

#define RANS_API extern "C" __attribute__((visibility("default")))

namespace rb {

int num_sms(int device) {
  static int cache[128] = {0};
  if (device < 0 || device >= 128) return 1;
  if (cache[device] == 0) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, device);
    cache[device] = v > 0 ? v : 1;
  }
  return cache[device];
}

int smem_optin(int device) {
  static int cache[128] = {0};
  if (device < 0 || device >= 128) return 0;
  if (cache[device] == 0) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, device);
    cache[device] = v;
  }
  return cache[device];
}

// Launch set-up answers cached per (kernel, device): the dynamic shared
// memory limit already set, and resident blocks per SM for a (threads,
// shared memory) pair, so a coding call repeats no runtime query.
namespace {
struct SmemEntry {
  const void *fn;
  int dev;
  uint32_t bytes;
};
struct OccEntry {
  const void *fn;
  int dev, threads;
  uint32_t smem;
  int blocks;
};
std::mutex g_launch_mutex;
std::vector<SmemEntry> g_smem_set;
std::vector<OccEntry> g_occ;
}  // namespace

cudaError_t ensure_dyn_smem(const void *fn, uint32_t bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_launch_mutex);
  for (SmemEntry &x : g_smem_set)
    if (x.fn == fn && x.dev == dev) {
      if (x.bytes >= bytes) return cudaSuccess;
      e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
      if (e == cudaSuccess) x.bytes = bytes;
      return e;
    }
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) g_smem_set.push_back({fn, dev, bytes});
  return e;
}

cudaError_t blocks_per_sm(int *out, const void *fn, int threads, uint32_t smem) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_launch_mutex);
  for (const OccEntry &x : g_occ)
    if (x.fn == fn && x.dev == dev && x.threads == threads && x.smem == smem) {
      *out = x.blocks;
      return cudaSuccess;
    }
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(out, fn, threads, (size_t)smem);
  if (e == cudaSuccess && g_occ.size() < 4096) g_occ.push_back({fn, dev, threads, smem, *out});
  return e;
}

}  // namespace rb

namespace {

using rb::Geom;

// An NVTX range around an entry point, so that traces show the library's
// calls (no cost beyond a call when no tool is attached).
struct NvtxRange {
  explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};

constexpr uint64_t kWsHeader = 256;

uint64_t align256(uint64_t v) { return (v + 255) & ~uint64_t(255); }

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

bool is_pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }

int make_geom(const rans_chunking *ch, int64_t n, Geom &g) {
  if (ch == nullptr || n < 0) return RANS_ERR_ARG;
  if (ch->interleave != 1 && ch->interleave != 2 && ch->interleave != 4 && ch->interleave != 8 &&
      ch->interleave != 32)
    return RANS_ERR_ARG;
  if (!is_pow2(ch->index_block)) return RANS_ERR_ARG;
  const int base_fmt = ch->format & ~RANS_FMT_ALIAS;
  const bool alias = (ch->format & RANS_FMT_ALIAS) != 0;
  if (base_fmt != RANS_FMT_RANS64 && base_fmt != RANS_FMT_RANS32_16) return RANS_ERR_ARG;
  if (alias && ch->interleave == 32) return RANS_ERR_ARG;  // no 32-way alias coder
  std::memset(&g, 0, sizeof(g));
  g.kind = ch->kind;
  g.fmt = base_fmt;
  g.alias = alias ? 1 : 0;
  g.W = ch->interleave;
  g.n = n;
  int ib = 0;
  while ((int64_t(1) << ib) < ch->index_block) ++ib;
  g.ib_shift = ib;
  g.slot_extra = 16ull * (uint64_t)g.W + 16ull;
  int64_t max_n = 0;
  switch (ch->kind) {
    case RANS_CHUNK_CONTIG:
      if (ch->n_streams < 1) return RANS_ERR_ARG;
      g.S = ch->n_streams;
      g.per = cdiv(n, g.S);
      max_n = g.per;
      if (g.per >= (int64_t(1) << 31) - 64) return RANS_ERR_ARG;
      break;
    case RANS_CHUNK_EXPLICIT:
      if (ch->n_streams < 0 || (ch->n_streams > 0 && ch->stream_starts == nullptr))
        return RANS_ERR_ARG;
      g.S = ch->n_streams;
      g.starts = ch->stream_starts;
      break;
    case RANS_CHUNK_TILED: {
      const int64_t B = ch->shape[0], C = ch->shape[1], H = ch->shape[2], W = ch->shape[3];
      if (B < 0 || C < 1 || H < 1 || W < 1) return RANS_ERR_ARG;
      if (ch->group < 1 || ch->tile_h < 1 || ch->tile_w < 1) return RANS_ERR_ARG;
      if (B * C * H * W != n) return RANS_ERR_ARG;
      g.C = C;
      g.H = H;
      g.Wd = W;
      g.cg = ch->group;
      g.th = ch->tile_h;
      g.tw = ch->tile_w;
      g.ng = cdiv(C, g.cg);
      g.nty = cdiv(H, g.th);
      g.ntx = cdiv(W, g.tw);
      g.S = B * g.ng * g.nty * g.ntx;
      max_n = (g.cg < C ? g.cg : C) * (g.th < H ? g.th : H) * (g.tw < W ? g.tw : W);
      if (C * H * W >= (int64_t(1) << 31) - 64) return RANS_ERR_ARG;
      {
        // tile classes (last group?, last tile row?, last tile column?), largest first
        const int64_t full[3] = {C % g.cg ? g.ng - 1 : g.ng, H % g.th ? g.nty - 1 : g.nty,
                                 W % g.tw ? g.ntx - 1 : g.ntx};
        const int64_t part[3] = {C % g.cg ? 1 : 0, H % g.th ? 1 : 0, W % g.tw ? 1 : 0};
        const int64_t fsz[3] = {g.cg, g.th, g.tw};
        const int64_t psz[3] = {C % g.cg, H % g.th, W % g.tw};
        int64_t size[8], count[8];
        int bits[8], nc = 0;
        for (int b = 0; b < 8; ++b) {
          int64_t cnt = B, sz = 1;
          for (int d = 0; d < 3; ++d) {
            cnt *= (b >> d & 1) ? part[d] : full[d];
            sz *= (b >> d & 1) ? psz[d] : fsz[d];
          }
          if (cnt == 0) continue;
          int at = nc++;
          while (at > 0 && size[at - 1] < sz) {  // stable insertion, larger first
            size[at] = size[at - 1];
            count[at] = count[at - 1];
            bits[at] = bits[at - 1];
            --at;
          }
          size[at] = sz;
          count[at] = cnt;
          bits[at] = b;
        }
        g.nclass = nc;
        int64_t run = 0;
        for (int i = 0; i < nc; ++i) {
          g.cls_start[i] = run;
          g.cls_bits[i] = bits[i];
          run += count[i];
        }
        if (run != g.S) return RANS_ERR_ARG;
      }
      break;
    }
    default:
      return RANS_ERR_ARG;
  }
  g.slot_bytes = rb::pad16(8ull * (uint64_t)max_n + g.slot_extra);
  return RANS_OK;
}

uint64_t lens_bytes(const Geom &g) { return align256(8ull * (uint64_t)g.S); }

uint64_t scratch_bytes(const Geom &g) {
  if (g.kind == RANS_CHUNK_EXPLICIT) return align256(8ull * (uint64_t)g.n + g.slot_extra * g.S);
  return align256(g.slot_bytes * (uint64_t)g.S);
}

uint64_t enc_ws_bytes(const Geom &g) { return kWsHeader + lens_bytes(g) + scratch_bytes(g); }

bool tables_usable(const rans_tables *t) {
  if (t == nullptr || t->blob == nullptr || t->K < 1) return false;
  if (t->precision < 1 || t->precision > 16) return false;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != t->device) return false;
  return true;
}

// RANS64 codes rows of precision 16, RANS32_16 rows of precision <= 15;
// alias coding needs the alias tables.
bool format_fits(const Geom &g, const rans_tables *t) {
  if (g.alias && t->alias == nullptr) return false;
  return g.fmt == RANS_FMT_RANS64 ? t->precision == 16 : t->precision <= 15;
}

// Bytes of the format's stream word.
uint64_t word_bytes(const Geom &g) { return g.fmt == RANS_FMT_RANS32_16 ? 2 : 4; }

cudaStream_t as_stream(void *s) { return static_cast<cudaStream_t>(s); }

}  // namespace

RANS_API const char *rans_status_string(int status) {
  switch (status) {
    case RANS_OK: return "ok";
    case RANS_ERR_ARG: return "invalid argument";
    case RANS_ERR_INDEX: return "index outside [0, K)";
    case RANS_ERR_ZERO_FREQ: return "symbol maps to a bucket of width 0";
    case RANS_ERR_RANGE: return "escape raw value of 2^60 or more";
    case RANS_ERR_CAPACITY: return "buffer too small";
    case RANS_ERR_CORRUPT: return "stream truncated, too long or inconsistent";
    case RANS_ERR_CUDA: return "CUDA runtime call failed";
    case RANS_ERR_TABLE: return "malformed CDF row or pmf";
    case RANS_ERR_TIMEOUT: return "bounded device wait gave up";
    default: return "unknown status";
  }
}

RANS_API int rans_version(void) { return 100; }

RANS_API int rans_gaussian_lengths(const float *scales, int32_t K, double tail_mass,
                                   int32_t *cdf_lengths, int32_t *offsets, void *stream) {
  if (K < 1 || !scales || !cdf_lengths || !offsets) return RANS_ERR_ARG;
  if (!(tail_mass > 0.0) || !(tail_mass < 1.0)) return RANS_ERR_ARG;
  return rb::launch_gaussian_lengths(scales, K, tail_mass, cdf_lengths, offsets,
                                     as_stream(stream));
}

RANS_API int rans_build_cdfs_from_scales(const float *scales, int32_t K, double tail_mass,
                                         int32_t precision, int32_t *cdfs, int32_t Lmax,
                                         int32_t *cdf_lengths, int32_t *offsets, void *stream) {
  NvtxRange nvtx_("rans_build_cdfs_from_scales");
  if (K < 1 || Lmax < 3 || !scales || !cdfs || !cdf_lengths || !offsets) return RANS_ERR_ARG;
  if (!(tail_mass > 0.0) || !(tail_mass < 1.0)) return RANS_ERR_ARG;
  if (precision < 1 || precision > 16) return RANS_ERR_ARG;
  return rb::launch_gaussian_rows(scales, K, tail_mass, precision, cdfs, Lmax, cdf_lengths,
                                  offsets, as_stream(stream));
}

RANS_API int rans_build_cdfs_from_pmfs(const float *pmfs, int32_t K, int32_t pmf_stride,
                                       const int32_t *pmf_lengths, const float *tail_mass,
                                       int32_t precision, int32_t *cdfs, int32_t Lmax,
                                       int32_t *cdf_lengths, void *stream) {
  NvtxRange nvtx_("rans_build_cdfs_from_pmfs");
  if (K < 1 || pmf_stride < 1 || Lmax < 2 || !pmfs || !pmf_lengths || !tail_mass || !cdfs ||
      !cdf_lengths)
    return RANS_ERR_ARG;
  if (precision < 1 || precision > 16) return RANS_ERR_ARG;
  return rb::launch_pmf_rows(pmfs, K, pmf_stride, pmf_lengths, tail_mass, precision, cdfs,
                             Lmax, cdf_lengths, as_stream(stream));
}

RANS_API uint64_t rans_tables_bytes(int32_t K, int32_t Lmax) {
  return rb::tables_bytes_bound(K, Lmax);
}

RANS_API int rans_tables_prepare(const int32_t *cdfs, int32_t K, int32_t Lmax,
                                 const int32_t *cdf_lengths, const int32_t *offsets,
                                 int32_t precision, void *blob, uint64_t blob_bytes,
                                 rans_tables *out, void *stream) {
  NvtxRange nvtx_("rans_tables_prepare");
  if (K < 1 || Lmax < 2 || Lmax > 65537 || !cdfs || !cdf_lengths || !offsets || !blob || !out)
    return RANS_ERR_ARG;
  if (precision < 1 || precision > 16) return RANS_ERR_ARG;
  return rb::prepare_tables(cdfs, K, Lmax, cdf_lengths, offsets, precision, blob, blob_bytes,
                            out, as_stream(stream));
}

RANS_API int rans_tables_refresh(const int32_t *cdfs, int32_t K, int32_t Lmax,
                                 const int32_t *cdf_lengths, const int32_t *offsets,
                                 const rans_tables *tables, void *stream) {
  NvtxRange nvtx_("rans_tables_refresh");
  if (!tables_usable(tables) || K != tables->K || Lmax < 2 || !cdfs || !cdf_lengths || !offsets)
    return RANS_ERR_ARG;
  return rb::refresh_tables(cdfs, K, Lmax, cdf_lengths, offsets, *tables, as_stream(stream));
}

RANS_API int rans_tables_refresh_from_scales(const float *scales, int32_t K, double tail_mass,
                                             int32_t *cdfs, int32_t Lmax, int32_t *cdf_lengths,
                                             int32_t *offsets, const rans_tables *tables,
                                             void *stream) {
  NvtxRange nvtx_("rans_tables_refresh_from_scales");
  if (!tables_usable(tables) || K != tables->K || Lmax < 3 || !scales || !cdfs ||
      !cdf_lengths || !offsets)
    return RANS_ERR_ARG;
  if (!(tail_mass > 0.0) || !(tail_mass < 1.0)) return RANS_ERR_ARG;
  return rb::refresh_tables_from_scales(scales, K, tail_mass, cdfs, Lmax, cdf_lengths, offsets,
                                        *tables, as_stream(stream));
}

RANS_API uint64_t rans_alias_bytes(const rans_tables *tables) {
  if (!tables || tables->K < 1 || tables->precision < 1 || tables->precision > 16) return 0;
  return ((8ull * (uint64_t)tables->n_buckets + 255) & ~255ull) +
         2ull * (uint64_t)tables->K * (1ull << tables->precision);
}

RANS_API int rans_alias_prepare(const int32_t *cdfs, int32_t K, int32_t Lmax,
                                const int32_t *cdf_lengths, rans_tables *tables, void *alias,
                                uint64_t alias_bytes, void *stream) {
  NvtxRange nvtx_("rans_alias_prepare");
  if (!tables_usable(tables) || K != tables->K || Lmax < 2 || !cdfs || !cdf_lengths || !alias)
    return RANS_ERR_ARG;
  return rb::prepare_alias(cdfs, K, Lmax, cdf_lengths, *tables, alias, alias_bytes,
                           as_stream(stream));
}

RANS_API int64_t rans_num_streams(const rans_chunking *chunking, int64_t n) {
  Geom g;
  int st = make_geom(chunking, n, g);
  return st ? st : g.S;
}

RANS_API uint64_t rans_encode_workspace_bytes(const rans_chunking *chunking, int64_t n) {
  Geom g;
  if (make_geom(chunking, n, g)) return 0;
  return enc_ws_bytes(g);
}

RANS_API uint64_t rans_decode_workspace_bytes(const rans_chunking *chunking, int64_t n) {
  Geom g;
  if (make_geom(chunking, n, g)) return 0;
  return kWsHeader;
}

RANS_API uint64_t rans_max_compressed_bytes(const rans_chunking *chunking, int64_t n) {
  Geom g;
  if (make_geom(chunking, n, g)) return 0;
  return 8ull * (uint64_t)n + g.slot_extra * (uint64_t)g.S;
}

RANS_API int rans_encode_with_indexes(const void *symbols, int32_t sym_dtype,
                                      const int32_t *indexes, int64_t n,
                                      const rans_tables *tables, const rans_chunking *chunking,
                                      uint8_t *out, uint64_t out_capacity,
                                      uint64_t *stream_offsets, void *workspace,
                                      uint64_t workspace_bytes, void *stream) {
  NvtxRange nvtx_("rans_encode_with_indexes");
  if (!tables_usable(tables)) return RANS_ERR_ARG;
  if (n > 0 && (!symbols || !indexes)) return RANS_ERR_ARG;
  if (!stream_offsets || !workspace || (out_capacity > 0 && !out)) return RANS_ERR_ARG;
  if (sym_dtype != RANS_SYM_INT32 && sym_dtype != RANS_SYM_UINT8 && sym_dtype != RANS_SYM_INT16)
    return RANS_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return RANS_ERR_ARG;
  Geom g;
  int st = make_geom(chunking, n, g);
  if (st) return st;
  if (!format_fits(g, tables)) return RANS_ERR_ARG;
  if (workspace_bytes < enc_ws_bytes(g)) return RANS_ERR_CAPACITY;
  cudaStream_t s = as_stream(stream);
  char *ws = reinterpret_cast<char *>(workspace);
  int32_t *status = reinterpret_cast<int32_t *>(ws);
  uint64_t *lens = reinterpret_cast<uint64_t *>(ws + kWsHeader);
  char *scratch = ws + kWsHeader + lens_bytes(g);
  if (cudaMemsetAsync(ws, 0, kWsHeader + 8ull * (uint64_t)g.S, s) != cudaSuccess)
    return RANS_ERR_CUDA;
  if (g.S > 0) {
    st = rb::launch_encode(symbols, sym_dtype, indexes, *tables, g, scratch, lens, status, s);
    if (st) return st;
  }
  return rb::launch_compact(g, scratch, lens, out, out_capacity, stream_offsets, status, s);
}

RANS_API int rans_decode_with_indexes(const uint8_t *in, uint64_t in_bytes,
                                      const uint64_t *stream_offsets, const int32_t *indexes,
                                      int64_t n, const rans_tables *tables,
                                      const rans_chunking *chunking, void *symbols_out,
                                      int32_t sym_dtype, void *workspace,
                                      uint64_t workspace_bytes, void *stream) {
  NvtxRange nvtx_("rans_decode_with_indexes");
  if (!tables_usable(tables)) return RANS_ERR_ARG;
  if (n > 0 && (!symbols_out || !indexes)) return RANS_ERR_ARG;
  if (!stream_offsets || !workspace || (in_bytes > 0 && !in)) return RANS_ERR_ARG;
  if (sym_dtype != RANS_SYM_INT32 && sym_dtype != RANS_SYM_UINT8 && sym_dtype != RANS_SYM_INT16)
    return RANS_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return RANS_ERR_ARG;
  Geom g;
  int st = make_geom(chunking, n, g);
  if (st) return st;
  if (!format_fits(g, tables)) return RANS_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(in) & (word_bytes(g) - 1)) != 0) return RANS_ERR_ARG;
  if (workspace_bytes < kWsHeader) return RANS_ERR_CAPACITY;
  cudaStream_t s = as_stream(stream);
  int32_t *status = reinterpret_cast<int32_t *>(workspace);
  if (cudaMemsetAsync(workspace, 0, kWsHeader, s) != cudaSuccess) return RANS_ERR_CUDA;
  if (g.S == 0) return RANS_OK;
  return rb::launch_decode(in, in_bytes, stream_offsets, indexes, *tables, g, symbols_out,
                           sym_dtype, status, s);
}

// ---- float latents ------------------------------------------------------

RANS_API int rans_build_indexes(const float *scales, int64_t n, const float *scale_table,
                                int32_t K, float scale_bound, int32_t *indexes, void *stream) {
  NvtxRange nvtx_("rans_build_indexes");
  if (n < 0 || K < 1 || (n > 0 && (!scales || !scale_table || !indexes))) return RANS_ERR_ARG;
  return rb::launch_build_indexes(scales, n, scale_table, K, scale_bound, indexes,
                                  as_stream(stream));
}

// The float entry points take one scale per element (index_block 1) and a
// scale table with one entry per table row.
static int float_args(const rans_tables *tables, const rans_chunking *chunking,
                      int32_t table_len) {
  if (!tables_usable(tables) || !chunking) return RANS_ERR_ARG;
  if (table_len != tables->K || chunking->index_block != 1) return RANS_ERR_ARG;
  if (chunking->format != RANS_FMT_RANS64 || tables->precision != 16) return RANS_ERR_ARG;
  if (chunking->interleave != 1 && chunking->interleave != 32) return RANS_ERR_ARG;
  return RANS_OK;
}

RANS_API int rans_encode_from_scales(const float *y, const float *means, const float *scales,
                                     int64_t n, const float *scale_table, int32_t table_len,
                                     float scale_bound, const rans_tables *tables,
                                     const rans_chunking *chunking, uint8_t *out,
                                     uint64_t out_capacity, uint64_t *stream_offsets,
                                     void *workspace, uint64_t workspace_bytes, void *stream) {
  NvtxRange nvtx_("rans_encode_from_scales");
  int st = float_args(tables, chunking, table_len);
  if (st) return st;
  if (n > 0 && (!y || !scales || !scale_table)) return RANS_ERR_ARG;
  if (!stream_offsets || !workspace || (out_capacity > 0 && !out)) return RANS_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return RANS_ERR_ARG;
  Geom g;
  st = make_geom(chunking, n, g);
  if (st) return st;
  if (workspace_bytes < enc_ws_bytes(g)) return RANS_ERR_CAPACITY;
  cudaStream_t s = as_stream(stream);
  char *ws = reinterpret_cast<char *>(workspace);
  int32_t *status = reinterpret_cast<int32_t *>(ws);
  uint64_t *lens = reinterpret_cast<uint64_t *>(ws + kWsHeader);
  char *scratch = ws + kWsHeader + lens_bytes(g);
  if (cudaMemsetAsync(ws, 0, kWsHeader + 8ull * (uint64_t)g.S, s) != cudaSuccess)
    return RANS_ERR_CUDA;
  if (g.S > 0) {
    st = rb::launch_encode_float(y, means, scales, scale_table, scale_bound, *tables, g,
                                 scratch, lens, status, s);
    if (st) return st;
  }
  return rb::launch_compact(g, scratch, lens, out, out_capacity, stream_offsets, status, s);
}

RANS_API int rans_decode_to_values(const uint8_t *in, uint64_t in_bytes,
                                   const uint64_t *stream_offsets, const float *scales,
                                   const float *means, int64_t n, const float *scale_table,
                                   int32_t table_len, float scale_bound,
                                   const rans_tables *tables, const rans_chunking *chunking,
                                   float *values, void *workspace, uint64_t workspace_bytes,
                                   void *stream) {
  NvtxRange nvtx_("rans_decode_to_values");
  int st = float_args(tables, chunking, table_len);
  if (st) return st;
  if (n > 0 && (!values || !scales || !scale_table)) return RANS_ERR_ARG;
  if (!stream_offsets || !workspace || (in_bytes > 0 && !in)) return RANS_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return RANS_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(in) & 3) != 0) return RANS_ERR_ARG;
  Geom g;
  st = make_geom(chunking, n, g);
  if (st) return st;
  if (workspace_bytes < kWsHeader) return RANS_ERR_CAPACITY;
  cudaStream_t s = as_stream(stream);
  int32_t *status = reinterpret_cast<int32_t *>(workspace);
  if (cudaMemsetAsync(workspace, 0, kWsHeader, s) != cudaSuccess) return RANS_ERR_CUDA;
  if (g.S == 0) return RANS_OK;
  return rb::launch_decode_float(in, in_bytes, stream_offsets, scales, means, scale_table,
                                 scale_bound, *tables, g, values, status, s);
}

RANS_API int rans_get_status(void *workspace, void *stream) {
  if (!workspace) return RANS_ERR_ARG;
  cudaStream_t s = as_stream(stream);
  rb::StatusWord sw;
  if (cudaMemcpyAsync(&sw, workspace, sizeof(sw), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return RANS_ERR_CUDA;
  if (sw.code != 0) {
    if (cudaMemsetAsync(workspace, 0, sizeof(sw), s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
      return RANS_ERR_CUDA;
  }
  return sw.code;
}

RANS_API int rans_debug_divide(const uint64_t *x, const uint32_t *f, int64_t n, uint64_t *q,
                               uint32_t *r, void *stream) {
  if (n < 0 || (n > 0 && (!x || !f || !q || !r))) return RANS_ERR_ARG;
  return rb::launch_debug_divide(x, f, n, q, r, as_stream(stream));
}
