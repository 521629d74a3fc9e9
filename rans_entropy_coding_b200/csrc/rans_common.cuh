// rans_common.cuh -- device-side building blocks shared by the librans_b200
// kernels: format constants, the prepared-table layout, stream geometry, the
// encoder's division step and error reporting.
//
// Format (page title + section): 64-bit state, 32-bit words, 16-bit CDF
// precision ("torch_ans 0.3.0", Usage, rans64 row); lower state bound 2^31;
// bypass pieces of 4 bits ("torch_ans 0.3.0", Low-level API, rans_push).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "rans_b200.h"

namespace rb {

constexpr uint32_t kPrec = 16;
constexpr uint32_t kTotal = 1u << kPrec;
constexpr uint64_t kL = 1ull << 31;            // state lower bound
constexpr uint32_t kBypassBits = 4;
constexpr uint32_t kBypassMax = 15;
constexpr unsigned kFull = 0xffffffffu;

// ------------------------------------------------------------ table blob --
// [header 256 B][RowMeta K x 8][bucket words][16-bit starts][slot words],
// sections 16-B padded.  The starts are the CDF entries mod 2^16 at the same
// indexes as the bucket words, plus one trailing 0: bucket j of a row ends at
// start[base + j + 1] (the next row's leading 0 stands for 65536).  Each row's metadata is stored 8 times side by side (128 bytes per
// row): lane l of a warp reads copy l mod 8, so the 8 lanes served by one
// shared-memory wavefront of 16-byte loads always hit 8 different bank groups.
// A bucket word packs start | (width - 1) << 16.
// Each row has 2^q slots (8 <= q <= 14) of width w = 2^(16-q) <= 256 over the
// cumulative range; a slot word packs lo | e1 << 16 | e2 << 24 where lo is the
// row-local bucket holding the slot's first cumulative value and e1, e2
// describe the bucket boundaries strictly inside the slot, as offsets from the
// slot start minus one (255 = none):
//   e1 <= e2:         at most two boundaries; for c = cum mod w the bucket is
//                     lo + (c > e1) + (c > e2);
//   e1 = 255 > e2:    three or more, resolved by boundary bitmaps: the 24-bit
//                     index p = lo | e2 << 16 (into the slot words) starts
//                     max(1, w / 16) bitmap words, word k covering cumulative
//                     values [16 k, 16 k + 16) of the slot as
//                     bits | j << 16, where j is the bucket holding the first
//                     value and bit i (1..15) marks a bucket starting i values
//                     later; the bucket is j + popc(bits & (2^(i+1) - 1));
//   255 > e1 > e2:    three or more with no bitmap room left (e2 + 3
//                     boundaries): a short binary search over the starts.
// Bitmap words follow the slots of all rows; the blob header counts the words
// handed out and flags whether any slot fell back to searching.
struct RowMeta {
  uint32_t bucket_base;  // index of the row's bucket 0 in the bucket words
  uint32_t maxv;         // escape bucket = cdf_length - 2
  int32_t offset;        // value of bucket 0
  uint32_t slot;         // slot base | (16 - q) << 27, q = log2(slots in row)
};
static_assert(sizeof(RowMeta) == 16, "RowMeta is one 16-byte load");
constexpr int kMetaCopies = 8;

__device__ __forceinline__ const RowMeta &row_meta(const RowMeta *meta, uint32_t r) {
  return meta[r * kMetaCopies + (threadIdx.x & (kMetaCopies - 1))];
}

constexpr uint32_t kHeaderBytes = 256;
constexpr uint32_t kChunkUsedWord = 16;    // header word: bitmap words handed out
constexpr uint32_t kSearchFlagWord = 17;   // header word: 1 if a slot searches
constexpr uint32_t kMaxChunkIndex = 0xff0000u;  // bitmap indexes fit lo | e2 << 16
constexpr int kMinQ = 8;
constexpr int kMaxQ = 14;

// Streaming inputs (row indexes, and int32 symbols when encoding) reach the
// warp coders through a per-warp shared-memory ring of groups filled with
// cp.async: one counting barrier tracks every copy in flight, so the
// registers' dependency barriers stay free for the serial state chain.
constexpr int kDecStage = 8;       // decoder ring: 8 groups of row indexes
constexpr int kEncStage = 16;      // encoder ring: 16 groups of indexes + symbols
constexpr int kDecMaxWarps = 24;   // decoder CTA: up to 768 threads
constexpr int kEncMaxWarps = 24;   // encoder CTA: up to 768 threads
constexpr uint32_t kDecStageBytes = kDecMaxWarps * kDecStage * 32 * 4;
// Tile-staged warp decoder: per warp a ring of two halves of 4 tile rows of
// up to 64 int32 each, 128-byte aligned.
constexpr uint32_t kTileRingHalf = 1024;
constexpr uint32_t kTileRingBytes = 2 * kTileRingHalf;
// The tile decoder's shared memory per stream: its index ring and a word
// window of the same size.
constexpr uint32_t kTileStreamBytes = 2 * kTileRingBytes;
// Shared memory the decoder's tables leave for its rings.
constexpr uint32_t kDecRingRoom = kDecMaxWarps * kTileRingBytes + 128;
static_assert(kDecRingRoom >= kDecStageBytes, "room for either decoder's rings");
// Streams a tile decoder CTA holds at once.
constexpr int kTileMaxStreams = (int)((kDecRingRoom - 128) / kTileStreamBytes);
constexpr uint32_t kEncStageBytes = kEncMaxWarps * kEncStage * 32 * 4 * 2;

__host__ __device__ inline uint64_t pad16(uint64_t b) { return (b + 15) & ~uint64_t(15); }

__device__ __forceinline__ uint32_t bucket_start(uint32_t e) { return e & 0xffffu; }
// width of a bucket from its start and the next start (mod 2^16; never 0)
__device__ __forceinline__ uint32_t width_of(uint32_t start, uint32_t next) {
  return ((next - start - 1u) & 0xffffu) + 1u;
}
__device__ __forceinline__ uint32_t bucket_freq(uint32_t e) { return (e >> 16) + 1u; }
__device__ __forceinline__ uint32_t slot_base(uint32_t s) { return s & 0x07ffffffu; }
__device__ __forceinline__ uint32_t slot_shift(uint32_t s) { return s >> 27; }

// ---------------------------------------------------------------- status --
// The first word of a workspace (and of a table blob's header) holds the
// first error recorded on the device; the second a detail (stream id).
struct StatusWord {
  int32_t code;
  int32_t pad;
  int64_t detail;
};

__device__ __forceinline__ void report(int32_t *status, int code, int64_t detail = 0) {
  if (atomicCAS(status, 0, code) == 0) {
    reinterpret_cast<StatusWord *>(status)->detail = detail;
  }
}

// ------------------------------------------------------------- geometry --
// Host-computed description of a chunking, passed by value to kernels.
struct Geom {
  int32_t kind;          // RANS_CHUNK_*
  int32_t W;             // 1, 2, 4, 8 or 32
  int64_t n;             // symbols
  int64_t S;             // streams
  int64_t per;           // CONTIG: ceil(n / S)
  const int64_t *starts; // EXPLICIT
  int64_t C, H, Wd;      // TILED tensor dims (batch is implied by S)
  int64_t cg, th, tw;    // TILED group / tile sizes
  int64_t ng, nty, ntx;  // TILED counts per image
  int32_t ib_shift;      // log2(index_block)
  int32_t nclass;        // TILED: tile classes in scheduling order (<= 8)
  int32_t fmt;           // RANS_FMT_RANS64 or RANS_FMT_RANS32_16
  int32_t alias;         // 1: alias-coded streams (RANS_FMT_ALIAS)
  uint64_t slot_bytes;   // CONTIG / TILED: uniform scratch slot per stream
  uint64_t slot_extra;   // 16 W + 16: per-stream scratch beyond 8 B/symbol
  // TILED: a class is the set of tiles sharing (last channel group?, last
  // tile row?, last tile column?); classes are listed largest tile first.
  int64_t cls_start[8];  // first work index of the class
  int32_t cls_bits[8];   // bit 0: last group, bit 1: last tile row, 2: last column
};

// One stream's extent.  Element i of a stream (coding order) sits at flat
// position base + rel(i), where rel(i) = c*plane + h*row + w for
// i = (c * hh + h) * ww + w.  A contiguous stream is the case hh = 1,
// ww = "infinite", plane = row = 0 (rel(i) = i).  rel() fits in 32 bits: the
// host checks C*H*W (tiled) and every stream length (contiguous) against 2^31.
struct Tile {
  int32_t hh, ww, plane, row;
};
constexpr int32_t kNoWrap = 0x7fffffff;

struct StreamDesc {
  int64_t n;
  int64_t base;
  Tile t;
  bool ok;
};

__device__ __forceinline__ StreamDesc stream_desc(const Geom &g, int64_t s) {
  StreamDesc d;
  d.ok = true;
  d.t.hh = 1;
  d.t.ww = kNoWrap;
  d.t.plane = 0;
  d.t.row = 0;
  if (g.kind == RANS_CHUNK_CONTIG) {
    int64_t a = s * g.per;
    a = a < g.n ? a : g.n;
    int64_t b = a + g.per;
    b = b < g.n ? b : g.n;
    d.base = a;
    d.n = b - a;
  } else if (g.kind == RANS_CHUNK_EXPLICIT) {
    int64_t a = g.starts[s], b = g.starts[s + 1];
    d.ok = (a >= 0) && (a <= b) && (b <= g.n) && (b - a < (int64_t(1) << 31) - 64);
    d.base = a;
    d.n = d.ok ? b - a : 0;
  } else {
    int64_t per_img = g.ng * g.nty * g.ntx;
    int64_t b = s / per_img;
    int64_t r = s - b * per_img;
    int64_t gi = r / (g.nty * g.ntx);
    int64_t r2 = r - gi * (g.nty * g.ntx);
    int64_t ty = r2 / g.ntx;
    int64_t tx = r2 - ty * g.ntx;
    int64_t c0 = gi * g.cg, h0 = ty * g.th, w0 = tx * g.tw;
    int64_t nc = g.C - c0 < g.cg ? g.C - c0 : g.cg;
    int64_t hh = g.H - h0 < g.th ? g.H - h0 : g.th;
    int64_t ww = g.Wd - w0 < g.tw ? g.Wd - w0 : g.tw;
    d.t.plane = (int32_t)(g.H * g.Wd);
    d.t.row = (int32_t)g.Wd;
    d.t.hh = (int32_t)hh;
    d.t.ww = (int32_t)ww;
    d.base = ((b * g.C + c0) * g.H + h0) * g.Wd + w0;
    d.n = nc * hh * ww;
  }
  return d;
}

// Work index k -> stream id, visiting streams in non-increasing length order
// (tiled: tile classes largest first; contiguous and explicit: as numbered).
// Warps take work indices in a stride that spreads consecutive indices over
// CTAs, so the long streams are shared out evenly over SMs and sub-partitions.
__device__ __forceinline__ int64_t stream_of(const Geom &g, int64_t k) {
  if (g.kind != RANS_CHUNK_TILED || g.nclass <= 1) return k;
  int ci = 0;
  while (ci + 1 < g.nclass && k >= g.cls_start[ci + 1]) ++ci;
  int64_t j = k - g.cls_start[ci];
  const int bits = g.cls_bits[ci];
  const int64_t ngs = (bits & 1) ? 1 : (g.C % g.cg ? g.ng - 1 : g.ng);
  const int64_t nys = (bits & 2) ? 1 : (g.H % g.th ? g.nty - 1 : g.nty);
  const int64_t nxs = (bits & 4) ? 1 : (g.Wd % g.tw ? g.ntx - 1 : g.ntx);
  const int64_t tx0 = j % nxs;
  j /= nxs;
  const int64_t ty0 = j % nys;
  j /= nys;
  const int64_t g0 = j % ngs;
  const int64_t b = j / ngs;
  const int64_t gi = (bits & 1) ? g.ng - 1 : g0;
  const int64_t ty = (bits & 2) ? g.nty - 1 : ty0;
  const int64_t tx = (bits & 4) ? g.ntx - 1 : tx0;
  return ((b * g.ng + gi) * g.nty + ty) * g.ntx + tx;
}

// Byte offset of stream s's scratch slot end (words are written downward).
__device__ __forceinline__ uint64_t slot_end(const Geom &g, const StreamDesc &d, int64_t s) {
  if (g.kind == RANS_CHUNK_EXPLICIT) {
    uint64_t before = (uint64_t)(d.base - g.starts[0]);
    return 8ull * (before + (uint64_t)d.n) + g.slot_extra * (uint64_t)(s + 1);
  }
  return g.slot_bytes * (uint64_t)(s + 1);
}

// A position inside a stream, stepped by +-k elements.
struct RelPos {
  int32_t c, h, w;
  __device__ __forceinline__ void init(const Tile &t, int32_t i) {
    if (t.ww == kNoWrap) {
      c = 0;
      h = 0;
      w = i;
    } else {
      const int32_t per = t.hh * t.ww;
      c = i / per;
      const int32_t rem = i - c * per;
      h = rem / t.ww;
      w = rem - h * t.ww;
    }
  }
  __device__ __forceinline__ int32_t rel(const Tile &t) const { return c * t.plane + h * t.row + w; }
  __device__ __forceinline__ void fwd(const Tile &t, int32_t k) {
    w += k;
    while (w >= t.ww) {
      w -= t.ww;
      if (++h >= t.hh) { h = 0; ++c; }
    }
  }
  __device__ __forceinline__ void back(const Tile &t, int32_t k) {
    w -= k;
    while (w < 0) {
      w += t.ww;
      if (--h < 0) { h = t.hh - 1; --c; }
    }
  }
};

// Incremental form of RelPos for the warp kernels: rel is kept up to date,
// stepping by +-k.  WIDE (tile width >= k, or a contiguous stream) needs at
// most one row wrap per step and runs branch-free; narrow tiles loop.
template <bool WIDE>
struct Stepper {
  int32_t w, h, rel;
  int32_t ww, hh, drow, dplane;  // drow = row - ww, dplane = plane - hh * row
  __device__ __forceinline__ void init(const Tile &t, int32_t i) {
    RelPos p;
    p.init(t, i);
    w = p.w;
    h = p.h;
    rel = p.rel(t);
    ww = t.ww;
    hh = t.hh;
    drow = t.row - t.ww;
    dplane = t.plane - t.hh * t.row;
  }
  __device__ __forceinline__ void fwd(int32_t k) {
    w += k;
    rel += k;
    if (WIDE) {
      const bool wr = w >= ww;
      w -= wr ? ww : 0;
      rel += wr ? drow : 0;
      h += wr ? 1 : 0;
      const bool cw = h >= hh;
      h = cw ? 0 : h;
      rel += cw ? dplane : 0;
    } else {
      while (w >= ww) {
        w -= ww;
        rel += drow;
        if (++h >= hh) {
          h = 0;
          rel += dplane;
        }
      }
    }
  }
  __device__ __forceinline__ void back(int32_t k) {
    w -= k;
    rel -= k;
    if (WIDE) {
      const bool wr = w < 0;
      w += wr ? ww : 0;
      rel -= wr ? drow : 0;
      h -= wr ? 1 : 0;
      const bool cw = h < 0;
      h = cw ? hh - 1 : h;
      rel -= cw ? dplane : 0;
    } else {
      while (w < 0) {
        w += ww;
        rel -= drow;
        if (--h < 0) {
          h = hh - 1;
          rel -= dplane;
        }
      }
    }
  }
};

// Hints that bring data towards L2 ahead of use (no effect on results);
// callers issue them only for addresses inside their own buffers.
__device__ __forceinline__ void prefetch_l2(const void *p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// Bulk L2 prefetch of [p, p + bytes) restricted to whole 16-byte units that
// lie inside [lo, hi) (cp.async.bulk.prefetch wants 16-byte alignment).
__device__ __forceinline__ void bulk_prefetch_l2(const char *lo, const char *hi, const char *p,
                                                 uint64_t bytes) {
  uintptr_t a = reinterpret_cast<uintptr_t>(p);
  uintptr_t b = a + bytes;
  const uintptr_t l = (reinterpret_cast<uintptr_t>(lo) + 15) & ~uintptr_t(15);
  const uintptr_t h = reinterpret_cast<uintptr_t>(hi) & ~uintptr_t(15);
  a = (a + 15) & ~uintptr_t(15);
  b &= ~uintptr_t(15);
  if (a < l) a = l;
  if (b > h) b = h;
  while (a < b) {
    uint32_t sz = (b - a) > 65536 ? 65536u : (uint32_t)(b - a);
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a), "r"(sz) : "memory");
    a += sz;
  }
}

// Stores through the global state space (st.global), so that the compiler
// knows they cannot touch shared memory and may move shared-memory loads
// across them.
__device__ __forceinline__ void st_global(uint32_t *p, uint32_t v) { __stcg(p, v); }
__device__ __forceinline__ void st_global(uint16_t *p, uint16_t v) { __stcg(p, v); }
__device__ __forceinline__ void st_global(int32_t *p, int32_t v) { __stcs(p, v); }
__device__ __forceinline__ void st_global(int16_t *p, int16_t v) { __stcs(p, v); }
__device__ __forceinline__ void st_global(uint8_t *p, uint8_t v) { __stcs(p, v); }
__device__ __forceinline__ void st_global(float *p, float v) { __stcs(p, v); }

// ------------------------------------------------------ float latents --
// For coders that start from float latents (a mean-scale model's y, means
// and scales) instead of int32 symbols and row indexes: the pages name
// CompressAI's build_indexes and symbol = round(y - mean) without spelling
// them out, so the library takes their plain reading.
//
// Row of a scale s: the first of the K table entries (increasing) that is
// >= max(s, bound), a NaN scale counting as the bound; the last row when none
// of the first K - 1 is.  An unrolled binary search with the same STEPS steps
// on every lane (2^STEPS > K - 1): pos counts the entries below s among the
// first K - 1.  The table is read with plain loads: the coders keep a copy in
// shared memory when it fits.
template <int STEPS>
__device__ __forceinline__ uint32_t scale_row(float s, const float *table, int K) {
  int pos = 0;
#pragma unroll
  for (int i = STEPS - 1; i >= 0; --i) {
    const int step = 1 << i;
    if (pos + step <= K - 1 && table[pos + step - 1] < s) pos += step;
  }
  return (uint32_t)pos;
}
// The search for any K <= 65536: 6 steps up to 65 entries (a uniform branch
// on K), else 16.
__device__ __forceinline__ uint32_t scale_row(float s, const float *table, int K) {
  return K - 1 < 64 ? scale_row<6>(s, table, K) : scale_row<16>(s, table, K);
}
__device__ __forceinline__ float bound_scale(float s, float bound) {
  return s >= bound ? s : bound;  // NaN fails the compare: the bound
}

// The same rows without a search, for tables of 2 to 64 strictly increasing,
// positive, finite entries (the first K - 1 counted) and a positive bound:
// positive floats order like their bit patterns, so key(s) = bits(s) >>
// shift is monotone, and with the shift chosen so that no two counted
// entries share a key, the entries below s are cnt[key(s)] (those of smaller
// keys) plus the one entry of s's own key if it is below s.  The counts of
// key k and k + 1 sit side by side in one 16-bit word (cnt2[k]), one word per
// key from the first entry's key to one past the last one's, in shared
// memory.  With a positive bound every scale the coders look up is positive
// (NaN counts as the bound).
constexpr uint32_t kScaleKeyWords = 1024;
constexpr uint32_t kScaleKeyBytes = 2 * kScaleKeyWords;

struct ScaleKeys {
  const uint16_t *cnt2;
  const float *tab;
  uint32_t shift, kmin;
  int32_t nk1;  // last valid key index
  // s > 0 (a scale raised to the positive bound)
  __device__ __forceinline__ uint32_t row(float s) const {
    int32_t k = (int32_t)(__float_as_uint(s) >> shift) - (int32_t)kmin;
    k = min(max(k, 0), nk1);
    const uint32_t w = cnt2[k];
    const uint32_t c = w & 0xffu, c1 = w >> 8;
    return c + ((c1 > c && tab[c] < s) ? 1u : 0u);
  }
};

// Builds the key counts for the K-entry table tab (shared memory) into cnt2
// (kScaleKeyBytes of shared memory); every thread of the block calls it
// (two barriers) and gets the same answer: false when the table or the
// bound does not qualify, and the coder then searches.
__device__ __forceinline__ bool build_scale_keys(const float *tab, int K, float bound,
                                                 uint16_t *cnt2, ScaleKeys &keys) {
  bool ok = K >= 2 && K <= 64 && bound > 0.0f;
  const float t0 = ok ? tab[0] : 1.0f, tl = ok ? tab[K - 2] : 1.0f;
  ok = ok && t0 > 0.0f && tl < INFINITY;
  const uint32_t b0 = __float_as_uint(t0), bl = __float_as_uint(tl);
  uint32_t shift = 0;
  while (shift < 31 && ((bl - b0) >> shift) + 2u > kScaleKeyWords - 1u) ++shift;
  const uint32_t kmin = b0 >> shift;
  const uint32_t nkeys = ok ? (bl >> shift) - kmin + 2u : 0u;
  for (int i = threadIdx.x; ok && i < K - 2; i += blockDim.x) {
    const float a = tab[i], b = tab[i + 1];
    ok = a < b && (__float_as_uint(a) >> shift) != (__float_as_uint(b) >> shift);
  }
  ok = __syncthreads_and(ok) != 0;
  if (ok) {
    for (uint32_t k = threadIdx.x; k < nkeys; k += blockDim.x) {
      uint32_t n0 = 0, n1 = 0;
      for (int i = 0; i <= K - 2; ++i) {
        const uint32_t ki = __float_as_uint(tab[i]) >> shift;
        n0 += ki < kmin + k;
        n1 += ki < kmin + k + 1;
      }
      cnt2[k] = (uint16_t)(n0 | (n1 << 8));
    }
  }
  __syncthreads();
  keys.cnt2 = cnt2;
  keys.tab = tab;
  keys.shift = shift;
  keys.kmin = kmin;
  keys.nk1 = (int32_t)nkeys - 1;
  return ok;
}

// Symbol of y given its mean: y - mean in float32, rounded to the nearest
// integer, ties to even.  ok is false (symbol 0) when it is not finite or not
// an int32.
__device__ __forceinline__ int32_t quantize(float y, float mean, bool &ok) {
  const float r = rintf(y - mean);
  ok = r >= -2147483648.0f && r < 2147483648.0f;
  return ok ? (int32_t)r : 0;
}

// ------------------------------------------------------------- symbols --
template <typename T> struct SymIO;
template <> struct SymIO<int32_t> {
  static __device__ __forceinline__ int32_t load(const void *p, int64_t i) {
    return __ldg(reinterpret_cast<const int32_t *>(p) + i);
  }
  static __device__ __forceinline__ void store(void *p, int64_t i, int64_t v) {
    reinterpret_cast<int32_t *>(p)[i] = (int32_t)v;
  }
};
template <> struct SymIO<int16_t> {
  static __device__ __forceinline__ int32_t load(const void *p, int64_t i) {
    return (int32_t)__ldg(reinterpret_cast<const short *>(p) + i);
  }
  static __device__ __forceinline__ void store(void *p, int64_t i, int64_t v) {
    reinterpret_cast<int16_t *>(p)[i] = (int16_t)v;
  }
};
template <> struct SymIO<uint8_t> {
  static __device__ __forceinline__ int32_t load(const void *p, int64_t i) {
    return (int32_t)__ldg(reinterpret_cast<const unsigned char *>(p) + i);
  }
  static __device__ __forceinline__ void store(void *p, int64_t i, int64_t v) {
    reinterpret_cast<uint8_t *>(p)[i] = (uint8_t)v;
  }
};

// ------------------------------------------------------------ cp.async --
__device__ __forceinline__ void cp_async4(void *smem_dst, const void *gsrc) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(
                   (uint32_t)__cvta_generic_to_shared(smem_dst)),
               "l"(gsrc)
               : "memory");
}
// 16 bytes, both addresses 16-byte aligned, bypassing L1.
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   (uint32_t)__cvta_generic_to_shared(smem_dst)),
               "l"(gsrc)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ------------------------------------------------------------- division --
// x / f and x % f for x < 2^47 f and 1 <= f <= 2^16 (so the quotient is below
// 2^47).  The quotient is estimated in double precision and corrected once in
// 32-bit integers (the "float divide + rarely taken exact integer fix-up" of
// "torch_ans 0.3.0", Performance Tuning, CPU item 3), branch-free:
//  * an unsigned 32-bit integer u becomes a double exactly as
//    (2^52 + u) - 2^52, with 2^52 + u assembled from its bit pattern (the
//    classical "magic number" conversion);
//  * x = xh 2^32 + xl is then formed with one fused multiply-add, rounded once
//    (relative error <= 2^-53);
//  * 1/f comes from the hardware reciprocal estimate refined by two
//    Newton-Raphson steps r <- r + r (1 - f r), each of which squares the
//    relative error (about 2^-52 after the second; a test divides exactly
//    for every f at the largest x);
//  * so q' = x * (1/f) is within 0.05 of the real quotient x/f; adding 2^52
//    rounds it to the nearest integer, which is floor(x/f) or one more, read
//    back from the low 52 bits of the sum;
//  * the remainder x - q f is then in [-f, f): it fits in 32 bits, and a
//    negative one means q was one too large.
__device__ __forceinline__ double u32_to_double(uint32_t u) {
  return __hiloint2double(0x43300000, (int)u) - 4503599627370496.0;  // 2^52
}

__device__ __forceinline__ double freq_reciprocal(uint32_t f) {
  const double fd = u32_to_double(f);
  double r;
  asm("rcp.approx.ftz.f64 %0, %1;" : "=d"(r) : "d"(fd));
#pragma unroll
  for (int i = 0; i < 2; ++i) r = fma(r, fma(-fd, r, 1.0), r);
  return r;
}

__device__ __forceinline__ void divmod_freq(uint64_t x, uint32_t f, double rcp, uint64_t &q,
                                            uint32_t &r) {
  const double xd =
      fma(u32_to_double((uint32_t)(x >> 32)), 4294967296.0, u32_to_double((uint32_t)x));
  const double t = fma(xd, rcp, 4503599627370496.0);  // 2^52 + round(x / f)
  uint64_t qe = (uint64_t)__double_as_longlong(t) & ((1ull << 52) - 1);
  const int32_t rem = (int32_t)((uint32_t)x - (uint32_t)qe * f);
  const bool over = rem < 0;
  q = qe - (over ? 1u : 0u);
  r = (uint32_t)(rem + (over ? (int32_t)f : 0));
}

// One symbol op of the encoder: x -> (x / f) 2^16 + x mod f + start.
__device__ __forceinline__ uint64_t enc_sym_step(uint64_t x, uint32_t start, uint32_t f,
                                                 double rcp) {
  uint64_t q;
  uint32_t r;
  divmod_freq(x, f, rcp, q, r);
  return (q << kPrec) + (r + start);
}

// The same division for a 32-bit state (x < 2^32 is exact in a double, so the
// argument above holds with room to spare).
__device__ __forceinline__ void divmod_freq32(uint32_t x, uint32_t f, double rcp, uint32_t &q,
                                              uint32_t &r) {
  const double t = fma(u32_to_double(x), rcp, 4503599627370496.0);  // 2^52 + round(x / f)
  const uint32_t qe = (uint32_t)__double_as_longlong(t);
  const int32_t rem = (int32_t)(x - qe * f);
  const bool over = rem < 0;
  q = qe - (over ? 1u : 0u);
  r = (uint32_t)(rem + (over ? (int32_t)f : 0));
}

// ------------------------------------------------------- coder formats --
// Two formats ("torch_ans 0.3.0", Usage, variants table):
//   Rans64: 64-bit state, 32-bit words, 16-bit precision, lower bound 2^31;
//   Rans32: 32-bit state, 16-bit words, precision p <= 15, lower bound 2^16
//           (the bound for which one 16-bit word restores the state).
// The prepared tables hold every CDF entry scaled to 16 bits (entry << sh,
// sh = 16 - p), so the lookup works on cum << sh and the coder shifts starts
// and widths back down.  In 16-bit units the renormalisation bound of either
// format is width16 * 2^(log2 L + word bits - 16): 2^47 and 2^16.
// A bypass op renormalises when x >= 2^(state bits - 5): 2^59 and 2^28.
struct Rans64 {
  using State = uint64_t;
  using Word = uint32_t;
  static constexpr uint32_t kWordBits = 32;
  static constexpr uint64_t kLow = 1ull << 31;
  static constexpr uint64_t kBitsBound = 1ull << 59;
  static constexpr int kFmt = RANS_FMT_RANS64;
  __device__ __forceinline__ static uint32_t shift(uint32_t) { return 0; }
  // x >= width16 * 2^47  <=>  high word of x >= width16 * 2^15
  __device__ __forceinline__ static bool need_word(uint64_t x, uint32_t f16) {
    return (uint32_t)(x >> 32) >= (f16 << 15);
  }
  __device__ __forceinline__ static double rcp(uint32_t f16, uint32_t) {
    return freq_reciprocal(f16);
  }
  __device__ __forceinline__ static uint64_t sym_step(uint64_t x, uint32_t start16, uint32_t f16,
                                                      double rcp, uint32_t) {
    return enc_sym_step(x, start16, f16, rcp);
  }
  // decoder: x -> width (x >> 16) + cum - start
  __device__ __forceinline__ static uint32_t cum16(uint64_t x, uint32_t) {
    return (uint32_t)x & (kTotal - 1);
  }
  __device__ __forceinline__ static uint64_t dec_step(uint64_t x, uint32_t cum16, uint32_t start16,
                                                      uint32_t f16, uint32_t) {
    return (uint64_t)f16 * (x >> kPrec) + (cum16 - start16);
  }
  // alias coding: the symbol's rank-th position from the row's remap
  // (encode), and x -> width (x >> 16) + rank (decode)
  __device__ __forceinline__ static uint64_t alias_step(uint64_t x, uint32_t start16, uint32_t f16,
                                                        double rcp, uint32_t,
                                                        const uint16_t *remap_row) {
    uint64_t q;
    uint32_t r;
    divmod_freq(x, f16, rcp, q, r);
    return (q << kPrec) + __ldg(remap_row + start16 + r);
  }
  __device__ __forceinline__ static uint64_t dec_rank_step(uint64_t x, uint32_t f16,
                                                           uint32_t rank, uint32_t) {
    return (uint64_t)f16 * (x >> kPrec) + rank;
  }
};

struct Rans32 {
  using State = uint32_t;
  using Word = uint16_t;
  static constexpr uint32_t kWordBits = 16;
  static constexpr uint32_t kLow = 1u << 16;
  static constexpr uint32_t kBitsBound = 1u << 28;
  static constexpr int kFmt = RANS_FMT_RANS32_16;
  __device__ __forceinline__ static uint32_t shift(uint32_t sh) { return sh; }
  __device__ __forceinline__ static bool need_word(uint32_t x, uint32_t f16) {
    return (x >> 16) >= f16;
  }
  __device__ __forceinline__ static double rcp(uint32_t f16, uint32_t sh) {
    return freq_reciprocal(f16 >> sh);
  }
  // x -> (x / f) 2^p + x mod f + start with f, start at precision p
  __device__ __forceinline__ static uint32_t sym_step(uint32_t x, uint32_t start16, uint32_t f16,
                                                      double rcp, uint32_t sh) {
    uint32_t q, r;
    divmod_freq32(x, f16 >> sh, rcp, q, r);
    return (q << (kPrec - sh)) + r + (start16 >> sh);
  }
  __device__ __forceinline__ static uint32_t cum16(uint32_t x, uint32_t sh) {
    return (x << sh) & (kTotal - 1);
  }
  __device__ __forceinline__ static uint32_t dec_step(uint32_t x, uint32_t cum16, uint32_t start16,
                                                      uint32_t f16, uint32_t sh) {
    return (f16 >> sh) * (x >> (kPrec - sh)) + ((cum16 - start16) >> sh);
  }
  __device__ __forceinline__ static uint32_t alias_step(uint32_t x, uint32_t start16, uint32_t f16,
                                                        double rcp, uint32_t sh,
                                                        const uint16_t *remap_row) {
    uint32_t q, r;
    divmod_freq32(x, f16 >> sh, rcp, q, r);
    return (q << (kPrec - sh)) + __ldg(remap_row + (start16 >> sh) + r);
  }
  __device__ __forceinline__ static uint32_t dec_rank_step(uint32_t x, uint32_t f16,
                                                           uint32_t rank, uint32_t sh) {
    return (f16 >> sh) * (x >> (kPrec - sh)) + rank;
  }
};

// ------------------------------------------------------------- alias ----
// Alias tables (a second blob, built by rans_alias_prepare): per row, slot
// words at the row's bucket indexes (bucket_base + j, slot j of the row's n
// = maxv + 1 slots of 2^p / n positions) packing d | (a | base << 16) << 32:
// positions [0, d) of the slot are the slot's own symbol j at ranks [0, d),
// the rest the alias symbol a at ranks base + (o - d); then 2^p 16-bit
// remap entries per row: remap[start + rank] = the position of that rank.
// The symbol and rank of position c (precision p) in row m.
__device__ __forceinline__ uint32_t alias_lookup(uint32_t c, const RowMeta &m,
                                                 const uint2 *slots, uint32_t prec,
                                                 uint32_t &rank) {
  const uint32_t log_n = 31 - __clz(m.maxv + 1);
  const uint32_t log_b = prec - log_n;
  const uint32_t j = c >> log_b;
  const uint32_t o = c & ((1u << log_b) - 1u);
  const uint2 e = __ldg(slots + m.bucket_base + j);
  const bool own = o < e.x;
  rank = own ? o : (e.y >> 16) + (o - e.x);
  return own ? j : (e.y & 0xffffu);
}

// ------------------------------------------------------- warp helpers --
__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// ------------------------------------------------ bulk staging (TMA) ----
// Copies `bytes` (multiple of 16, both addresses 16-B aligned) from global
// into shared memory with one-dimensional bulk copies (cp.async.bulk, no
// multicast) completing on an mbarrier.  The wait is bounded; on timeout the
// status gets RANS_ERR_TIMEOUT and false is returned.
__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(1000u)
      : "memory");
  return ok != 0;
}

__device__ inline bool stage_to_smem(void *dst, const void *src, uint32_t bytes,
                                     uint64_t *bar_storage, int32_t *status,
                                     void *dst2 = nullptr, const void *src2 = nullptr,
                                     uint32_t bytes2 = 0) {
  const uint32_t bar = smem_addr(bar_storage);
  if (threadIdx.x == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
                 "r"(bytes + bytes2)
                 : "memory");
    const uint32_t chunk = 32768;
    for (int part = 0; part < 2; ++part) {
      const char *s = reinterpret_cast<const char *>(part ? src2 : src);
      const uint32_t d = smem_addr(part ? dst2 : dst);
      const uint32_t nb = part ? bytes2 : bytes;
      for (uint32_t off = 0; off < nb; off += chunk) {
        uint32_t sz = nb - off < chunk ? nb - off : chunk;
        asm volatile(
            "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, "
            "[%3];" ::"r"(d + off),
            "l"(s + off), "r"(sz), "r"(bar)
            : "memory");
      }
    }
  }
  bool done = false;
  for (uint32_t it = 0; it < (1u << 21); ++it) {
    if (mbar_try_wait(bar, 0)) { done = true; break; }
  }
  if (!done) {
    report(status, RANS_ERR_TIMEOUT, -1);
    for (uint32_t it = 0; it < (1u << 21); ++it)
      if (mbar_try_wait(bar, 0)) break;
  }
  __syncthreads();
  return __syncthreads_and(done ? 1 : 0) != 0;
}

}  // namespace rb

// ------------------------------------------- tensor-tile staging (TMA) ----
// Tiles of an int32 tensor move between global and shared memory with
// cp.async.bulk.tensor (no multicast): a load completes on an mbarrier with a
// byte count, a store is tracked by the issuing thread's bulk groups.  The
// tensor maps (CUtensorMap, built on the host) describe a 3-D int32 tensor
// (x = width, y = height, z = image * channel) and a box of w x 4 rows x 1.
namespace rb {
namespace tma {

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void arrive_expect(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
// Orders this thread's generic-proxy shared-memory accesses before later
// async-proxy (bulk copy) accesses of the same memory.
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void load_3d(uint32_t dst, const void *map, int32_t x, int32_t y,
                                        int32_t z, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void store_3d(const void *map, int32_t x, int32_t y, int32_t z,
                                         uint32_t src) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%1, %2, %3}], [%4];" ::
          "l"(reinterpret_cast<uint64_t>(map)),
      "r"(x), "r"(y), "r"(z), "r"(src)
      : "memory");
}
// Brings a tensor tile into L2 ahead of its load (no completion to wait for).
__device__ __forceinline__ void prefetch_l2_3d(const void *map, int32_t x, int32_t y, int32_t z) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(z)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Waits until this thread's committed bulk stores have read their source.
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Waits until this thread's committed bulk stores have completed.
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
// Predicated forms (no branch around them): the operation runs only where p
// is nonzero, so a warp-wide code block can issue it from one lane.
__device__ __forceinline__ void arrive_expect_if(uint32_t p, uint32_t bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %0, 0;\n\t"
      "@q mbarrier.arrive.expect_tx.shared::cta.b64 _, [%1], %2;\n\t}" ::"r"(p),
      "r"(bar), "r"(bytes)
      : "memory");
}
__device__ __forceinline__ void load_3d_if(uint32_t p, uint32_t dst, const void *map, int32_t x,
                                           int32_t y, int32_t z, uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %0, 0;\n\t"
      "@q cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%1], [%2, {%3, %4, %5}], [%6];\n\t}" ::"r"(p),
      "r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void prefetch_l2_3d_if(uint32_t p, const void *map, int32_t x,
                                                  int32_t y, int32_t z) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %0, 0;\n\t"
      "@q cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%1, {%2, %3, %4}];\n\t}" ::"r"(p),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z)
      : "memory");
}
__device__ __forceinline__ void store_3d_commit_if(uint32_t p, const void *map, int32_t x,
                                                   int32_t y, int32_t z, uint32_t src) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %0, 0;\n\t"
      "@q cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%1, {%2, %3, %4}], [%5];"
      "\n\t@q cp.async.bulk.commit_group;\n\t}" ::"r"(p),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(src)
      : "memory");
}
__device__ __forceinline__ void bulk_wait_read_if(uint32_t p) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %0, 0;\n\t"
      "@q cp.async.bulk.wait_group.read 0;\n\t}" ::"r"(p)
      : "memory");
}

// A plain (1-D) bulk store of `bytes` bytes (a multiple of 16, both
// addresses 16-byte aligned) from shared to global memory, committed as one
// bulk group, where p is nonzero.
__device__ __forceinline__ void store_1d_commit_if(uint32_t p, void *dst, uint32_t src,
                                                   uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %0, 0;\n\t"
      "@q cp.async.bulk.global.shared::cta.bulk_group [%1], [%2], %3;"
      "\n\t@q cp.async.bulk.commit_group;\n\t}" ::"r"(p),
      "l"(reinterpret_cast<uint64_t>(dst)), "r"(src), "r"(bytes)
      : "memory");
}
// Waits, where p is nonzero, until every bulk group but the most recent one
// has read its shared-memory source.
__device__ __forceinline__ void bulk_wait_read1_if(uint32_t p) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %0, 0;\n\t"
      "@q cp.async.bulk.wait_group.read 1;\n\t}" ::"r"(p)
      : "memory");
}

// A bounded wait for phase `parity` of an mbarrier: true once it completed,
// false after `tries` attempts (each suspending for up to about 1 us).
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, uint32_t tries) {
  for (uint32_t it = 0; it < tries; ++it)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

}  // namespace tma
}  // namespace rb
