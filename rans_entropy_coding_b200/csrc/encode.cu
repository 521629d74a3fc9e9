// encode.cu -- encode_with_indexes: every stream is coded in reverse symbol
// order into a worst-case scratch slot (words written downward, the way a
// ryg_rans encoder fills its buffer from the end), then the streams are
// compacted behind a device prefix scan.  Tiled streams take their row
// indexes and symbols in as tensor-tile copies (encode_tile_kernel),
// contiguous streams of whole 256-symbol chunks with a row per chunk their
// symbols as 16-byte cp.async copies (encode_chunk_kernel); the general
// kernel streams both through a per-warp cp.async ring.
//
//  * value mapping and escape ("torch_ans 0.3.0", Low-level API, rans_push:
//    coded range [offset, offset + cdf_size - 2), zig-zag raw value, bypass
//    pieces; "kompressor" README, Correctness: the bypass path);
//  * symbol op: renormalise when x >= 2^47 freq, then
//    x = (x / freq) 2^16 + x mod freq + start (64-bit state, 32-bit words,
//    16-bit precision: "torch_ans 0.3.0", Usage, rans64 row); or, for the
//    rans32_16 format (same table, rans32_16 row), renormalise when
//    x >= 2^(32-p) freq and x = (x / freq) 2^p + x mod freq + start with
//    16-bit words and a 32-bit state (the F template parameter; see
//    Rans64 / Rans32 in rans_common.cuh);
//  * W = 32: one warp per stream, lane = symbol index mod 32, one shared word
//    stream ("torch_ans 0.3.0", Usage legend: __ballot_sync-based warp
//    renormalisation with one shared cursor; FAQ: interleaved states share
//    one bitstream, processed sequentially).  In the serial order a group of
//    32 symbols is coded lane 31 first, so lane l's words land below those of
//    lanes > l: a ballot + popc places them.  A group holding an escape is
//    coded off the fast path: each lane counts its words, a suffix sum over
//    lanes places them, and the lane writes them.
#include <type_traits>

#include <cuda.h>  // CUtensorMap

#include "rans_common.cuh"
#include "rans_internal.h"

namespace rb {
namespace {

constexpr int kEncThreads32 = kEncMaxWarps * 32;

// Per-warp ring: 16 groups of row indexes and symbols, or for float latents
// 8 groups of scales, y and means (the same shared memory budget).
__host__ __device__ constexpr int enc_ring_groups(bool flt) { return flt ? 8 : kEncStage; }
__host__ __device__ constexpr uint32_t enc_stage_bytes_per_warp(bool flt) {
  return (uint32_t)enc_ring_groups(flt) * 32u * 4u * (flt ? 3u : 2u);
}
static_assert(enc_stage_bytes_per_warp(true) <= enc_stage_bytes_per_warp(false),
              "the float ring fits the shared memory the tables leave for rings");
constexpr int kEncThreads1 = 128;

struct EncCtx {
  const void *sym;
  const int32_t *idx;
  // float latents instead of sym / idx (one scale per element): y, means
  // (or null), scales, the K-entry scale table, its lower bound
  const float *fy, *fmean, *fscale, *stab;
  float bound;
  int32_t stab_smem; // 1: the kernel copies the scale table into shared memory
  int32_t K;
  uint32_t sh;       // 16 - precision of the rows (Rans32; 0 for Rans64)
  const uint16_t *remap;  // alias coding: 2^p remap entries per row
  uint32_t meta_bytes, bucket_bytes, start_bytes;
  const char *blob;
  Geom g;
  char *scratch;
  uint64_t *lens;
  int32_t *status;
};

// Table modes of the encoder: 32-bit bucket words (start | (width - 1) <<
// 16), or, for tables too large to stage those, the 16-bit starts (a bucket's
// width is the distance to the next start).  bucket_word<ST> reads bucket i
// of the table `tab` in either form.
template <bool ST>
__device__ __forceinline__ uint32_t bucket_word(const uint32_t *tab, uint32_t i) {
  if (!ST) return tab[i];
  const uint16_t *starts = reinterpret_cast<const uint16_t *>(tab);
  const uint32_t a = starts[i], b = starts[i + 1];
  return a | (((b - a - 1u) & 0xffffu) << 16);
}

// Maps symbol s through row m: bucket start / width, and the escape's raw
// value (zig-zag: below the range 2|v| - 1, above it 2 (v - maxv)).
template <bool ST>
__device__ __forceinline__ void map_symbol(int32_t s, const RowMeta &m, const uint32_t *buckets,
                                           uint32_t &start, uint32_t &freq, uint64_t &raw,
                                           bool &esc) {
  int64_t v = (int64_t)s - (int64_t)m.offset;
  const int64_t maxv = (int64_t)m.maxv;
  raw = 0;
  if (v < 0) {
    raw = (uint64_t)(-2 * v - 1);
    v = maxv;
  } else if (v >= maxv) {
    raw = (uint64_t)(2 * (v - maxv));
    v = maxv;
  }
  esc = (v == maxv);
  const uint32_t e = bucket_word<ST>(buckets, m.bucket_base + (uint32_t)v);
  start = bucket_start(e);
  freq = bucket_freq(e);
}

// Bypass op: renormalise when x >= 2^59 (Rans32: 2^28), then append 4 bits.
template <class F, bool WRITE>
__device__ __forceinline__ void bits_op(typename F::State &x, uint32_t val,
                                        typename F::Word *end, uint32_t &k, uint32_t pos0) {
  if (x >= F::kBitsBound) {
    if (WRITE) st_global(end - 1 - (pos0 + k), (typename F::Word)x);
    ++k;
    x >>= F::kWordBits;
  }
  x = (x << kBypassBits) | val;
}

// All ops of one symbol, in reverse op order (bypass pieces last to first,
// then the count pieces last to first, then the symbol op).  Returns the
// number of words pushed; with WRITE they go to end[-1 - (pos0 + j)].
template <class F, bool WRITE, bool ALIAS = false>
__device__ __forceinline__ uint32_t symbol_ops(typename F::State &x, uint32_t start,
                                               uint32_t freq, double rcp, uint64_t raw, bool esc,
                                               typename F::Word *end, uint32_t pos0,
                                               uint32_t sh, const uint16_t *remap_row = nullptr) {
  uint32_t k = 0;
  if (esc) {
    uint32_t nb = 0;
    while (nb < 16 && (raw >> (kBypassBits * nb)) != 0) ++nb;
    for (int j = (int)nb - 1; j >= 0; --j)
      bits_op<F, WRITE>(x, (uint32_t)(raw >> (kBypassBits * j)) & kBypassMax, end, k, pos0);
    bits_op<F, WRITE>(x, nb % kBypassMax, end, k, pos0);
    for (uint32_t t = 0; t < nb / kBypassMax; ++t)
      bits_op<F, WRITE>(x, kBypassMax, end, k, pos0);
  }
  if (F::need_word(x, freq)) {
    if (WRITE) st_global(end - 1 - (pos0 + k), (typename F::Word)x);
    ++k;
    x >>= F::kWordBits;
  }
  if constexpr (ALIAS) x = F::alias_step(x, start, freq, rcp, sh, remap_row);
  else x = F::sym_step(x, start, freq, rcp, sh);
  return k;
}


// A group holding an escape, off the fast path: every lane counts the words
// its ops push, a suffix sum over lanes places each lane's block (lanes > l
// push first in the serial order), then each lane writes its words.
template <class F>
__device__ __forceinline__ typename F::State escape_group_enc(
    typename F::State x, bool active, uint32_t start, uint32_t freq, double rcp, uint64_t raw,
    bool esc, typename F::Word *end, uint32_t cursor, uint32_t &total, uint32_t sh) {
  const int lane = threadIdx.x & 31;
  uint32_t k = 0;
  if (active) {
    typename F::State y = x;
    k = symbol_ops<F, false>(y, start, freq, rcp, raw, esc, end, 0, sh);
  }
  uint32_t inc = k;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_down_sync(kFull, inc, o);
    if (lane + o < 32) inc += t;
  }
  total = __shfl_sync(kFull, inc, 0);
  if (active) symbol_ops<F, true>(x, start, freq, rcp, raw, esc, end, cursor + inc - k, sh);
  return x;
}

// Per-warp encoder state for one stream.
template <class F>
struct WarpEnc {
  typename F::State x;  // this lane's state
  uint32_t cursor;   // words pushed so far (written at end[-1 - k])
  uint32_t rmax;     // largest row index seen (checked once per stream)
  bool range_err;
};

// A group's table lookups, done one group ahead of its state update: they
// do not depend on the state, so they run while the previous group's
// division does.  The shared-memory read comes first (enc_bucket), the
// arithmetic on it later (enc_look), with the other group's state update in
// between.
struct EncLook {
  uint32_t start, freq;
  double rcp;
  int64_t v;         // s - offset (escape path)
  uint32_t maxv;
  bool esc;          // this lane escapes
  bool any_esc;      // some lane of the group escapes
};

struct EncBucket {
  uint32_t e;        // bucket word
  int64_t v;
  uint32_t maxv;
  bool in_range;
};

// value mapping: in range iff 0 <= s - offset < maxv (64-bit, exact)
template <bool ST>
__device__ __forceinline__ EncBucket enc_bucket(int32_t sv, const RowMeta &m,
                                                const uint32_t *buckets) {
  EncBucket b;
  b.v = (int64_t)sv - (int64_t)m.offset;
  b.maxv = m.maxv;
  b.in_range = (uint64_t)b.v < (uint64_t)m.maxv;
  b.e = bucket_word<ST>(buckets, m.bucket_base + (b.in_range ? (uint32_t)b.v : m.maxv));
  return b;
}

template <class F>
__device__ __forceinline__ EncLook enc_look(const EncBucket &b, bool active, uint32_t sh) {
  EncLook L;
  L.v = b.v;
  L.maxv = b.maxv;
  L.start = bucket_start(b.e);
  L.freq = bucket_freq(b.e);
  L.rcp = F::rcp(L.freq, sh);
  L.esc = active && !b.in_range;
  L.any_esc = __any_sync(kFull, L.esc);
  return L;
}

// One group of 32 symbols with no escape, coded lane 31 first: lanes whose
// state reaches the renormalisation bound push its low word (ballot + popc
// place the words), then every lane takes its symbol op.
template <class F, bool FULL>
__device__ __forceinline__ void enc_group_fast(WarpEnc<F> &st, const EncLook &L, bool active,
                                               uint32_t above, typename F::Word *end,
                                               uint32_t sh) {
  if (FULL) active = true;
  typename F::State x = st.x;
  const bool need = active && F::need_word(x, L.freq);
  const uint32_t bm = __ballot_sync(kFull, need);
  if (need) st_global(end - 1 - (st.cursor + __popc(bm & above)), (typename F::Word)x);
  x = need ? (x >> F::kWordBits) : x;
  st.cursor += __popc(bm);
  const typename F::State y = F::sym_step(x, L.start, L.freq, L.rcp, sh);
  st.x = active ? y : x;
}

// The same group holding an escape, from the state and cursor before it.
template <class F>
__device__ __forceinline__ void enc_group_escape(WarpEnc<F> &st, typename F::State x0,
                                                 uint32_t cursor0, const EncLook &L, bool active,
                                                 typename F::Word *end, uint32_t sh) {
  uint64_t raw = 0;
  if (L.esc) raw = L.v < 0 ? (uint64_t)(-2 * L.v - 1) : (uint64_t)(2 * (L.v - (int64_t)L.maxv));
  st.range_err |= L.esc && (raw >> 60) != 0;
  uint32_t total;
  st.x = escape_group_enc<F>(x0, active, L.start, L.freq, L.rcp, raw & ((1ull << 60) - 1),
                             L.esc, end, cursor0, total, sh);
  st.cursor = cursor0 + total;
}

// One warp codes one stream.  Per coded group k the loop runs, in this
// order: group k+1's bucket read, group k's state update, group k+1's
// reciprocal, then the copies for group k + kEncStage - 1 and the ring reads
// of groups k+2 (symbols, row metadata) and k+3 (row index); group k's rare
// escape path comes last.  Nothing in group k's state chain waits on a
// memory access issued in the same iteration.
// FLT: the stream's inputs are float latents: an 8-group ring holds scales
// (as the row source), y and the means; each group's row is its scale's
// table row and its symbol rint(y - mean).
template <class F, typename SymT, bool IB0, bool WIDE, bool FLT, bool ST>
__device__ __forceinline__ void encode_stream_w32(const EncCtx &c, const StreamDesc &d,
                                                  const RowMeta *meta, const uint32_t *buckets,
                                                  uint32_t *stg, int64_t s, const float *stab) {
  constexpr bool kStageSym = FLT || sizeof(SymT) == 4;
  constexpr int kS = enc_ring_groups(FLT);
  using Word = typename F::Word;
  const int lane = threadIdx.x & 31;
  Word *end = reinterpret_cast<Word *>(c.scratch + slot_end(c.g, d, s));
  const uint32_t sh = F::shift(c.sh);
  const int32_t n = (int32_t)d.n;
  const int32_t G = (n + 31) >> 5;
  const int64_t base = d.base;
  const int ib = c.g.ib_shift;
  const int32_t *idx_s = c.idx + (IB0 ? base : 0);
  const SymT *sym_s = reinterpret_cast<const SymT *>(c.sym) + base;
  const uint32_t kmax = (uint32_t)c.K - 1u;
  const uint32_t above = 0xfffffffeu << lane;   // lanes > this lane
  uint32_t *stg_idx = stg;
  uint32_t *stg_sym = stg + kS * 32;
  uint32_t *stg_mean = stg + 2 * kS * 32;  // FLT
  WarpEnc<F> st;
  st.x = F::kLow;
  st.cursor = 0;
  st.rmax = 0;
  st.range_err = false;

  // The k-th coded group (group G-1-k) lands in stage slot k mod kS, copied
  // kS - 1 groups ahead.  Copies for groups past the end (and lanes without
  // an element) read the stream's element 0, never used.  Narrow symbols are
  // read with plain loads one group ahead of use, after an L2 prefetch issued
  // with the copies.
  Stepper<WIDE> pl;
  pl.init(d.t, (G - 1) * 32 + lane);
  Stepper<WIDE> pn = pl;  // narrow symbols: position of the next load
  const float *fy_s = FLT ? c.fy + base : nullptr;
  const float *fs_s = FLT ? c.fscale + base : nullptr;
  const float *fm_s = FLT && c.fmean ? c.fmean + base : nullptr;
  auto issue = [&](int32_t ki) {
    const int32_t g = G - 1 - ki;
    const int32_t rel = ki < G && lane < n - g * 32 ? pl.rel : 0;
    const int slot = (ki & (kS - 1)) * 32 + lane;
    if (FLT) {
      cp_async4(stg_idx + slot, fs_s + rel);
      cp_async4(stg_sym + slot, fy_s + rel);
      if (fm_s) cp_async4(stg_mean + slot, fm_s + rel);
    } else {
      cp_async4(stg_idx + slot, IB0 ? idx_s + rel : c.idx + ((base + rel) >> ib));
      if (kStageSym) cp_async4(stg_sym + slot, sym_s + rel);
      else prefetch_l2(sym_s + rel);
    }
    cp_async_commit();
    pl.back(32);
  };
  // FLT: the row of a staged scale, and the symbol of a staged y with its
  // mean (an out-of-range value is recorded and coded as 0)
  auto row_of = [&](uint32_t v) -> uint32_t {
    if (!FLT) return v;
    return scale_row(bound_scale(__uint_as_float(v), c.bound), stab, c.K);
  };
  auto quant = [&](int32_t ybits, float mean) -> int32_t {
    bool ok;
    const int32_t q = quantize(__int_as_float(ybits), mean, ok);
    st.range_err |= !ok;
    return q;
  };
  // FLT: the mean of coded group ki's element (from the ring, like y)
  auto mean_of = [&](int32_t ki) -> float {
    return fm_s ? __uint_as_float(stg_mean[(ki & (kS - 1)) * 32 + lane]) : 0.0f;
  };
  auto ring = [&](int32_t ki) { return (ki & (kS - 1)) * 32 + lane; };
  auto meta_of = [&](uint32_t r) -> RowMeta {
    st.rmax = max(st.rmax, r);
    return row_meta(meta, min(r, kmax));
  };
  // symbols of coded group ki (ki < G), from the ring or a plain load
  auto sym_of = [&](int32_t ki) -> int32_t {
    if (kStageSym) return (int32_t)stg_sym[ring(ki)];
    const int32_t v = SymIO<SymT>::load(sym_s, ki < G ? pn.rel : 0);
    pn.back(32);
    return v;
  };
#pragma unroll 1
  for (int32_t u = 0; u < kS - 1; ++u) issue(u);
  cp_async_wait<kS - 4>();  // coded groups 0..2 have landed
  // group G - 1 (coded first) may be partial
  const bool active0 = lane < n - (G - 1) * 32;
  int32_t s0;
  if (FLT) {
    s0 = active0 ? quant(sym_of(0), mean_of(0)) : 0;
  } else if (kStageSym) {
    s0 = sym_of(0);
  } else {
    s0 = SymIO<SymT>::load(sym_s, active0 ? pn.rel : 0);
    pn.back(32);
  }
  EncLook L =
      enc_look<F>(enc_bucket<ST>(s0, meta_of(row_of(stg_idx[ring(0)])), buckets), active0, sh);
  // group 1's symbol (FLT: its y and mean, quantised when used)
  int32_t s1 = G > 1 ? sym_of(1) : 0;
  float mean1 = FLT && G > 1 ? mean_of(1) : 0.0f;
  RowMeta m1 = meta_of(G > 1 ? row_of(stg_idx[ring(1)]) : 0u);
  uint32_t r2 = G > 2 ? row_of(stg_idx[ring(2)]) : 0u;

  auto step = [&](int32_t k, bool active, auto full) {
    // group k+1's bucket (after the last group: row 0, unused)
    if (FLT) s1 = k + 1 < G ? quant(s1, mean1) : 0;
    const EncBucket b1 = enc_bucket<ST>(s1, m1, buckets);
    // group k's state update
    const typename F::State x0 = st.x;
    const uint32_t c0 = st.cursor;
    enc_group_fast<F, decltype(full)::value>(st, L, active, above, end, sh);
    // group k+1's reciprocal and escape ballot
    const EncLook L1 = enc_look<F>(b1, true, sh);
    // copies, then the ring reads two and three groups ahead
    issue(k + kS - 1);
    cp_async_wait<kS - 4>();  // coded groups up to k + 3 have landed
    const int32_t s2 = k + 2 < G ? sym_of(k + 2) : 0;
    const float mean2 = FLT && k + 2 < G ? mean_of(k + 2) : 0.0f;
    const RowMeta m2 = meta_of(r2);
    const uint32_t r3 = k + 3 < G ? row_of(stg_idx[ring(k + 3)]) : 0u;
    if (L.any_esc) enc_group_escape<F>(st, x0, c0, L, active, end, sh);
    L = L1;
    s1 = s2;
    mean1 = mean2;
    m1 = m2;
    r2 = r3;
  };
  step(0, active0, std::false_type());
#pragma unroll 2
  for (int32_t k = 1; k < G; ++k) step(k, true, std::true_type());
  cp_async_wait<0>();
  if (__any_sync(kFull, st.rmax > kmax)) {
    if (lane == 0) report(c.status, RANS_ERR_INDEX, s);
    return;
  }
  if (__any_sync(kFull, st.range_err)) {
    if (lane == 0) report(c.status, RANS_ERR_RANGE, s);
    return;
  }
  // flush: lanes 31..0 push high then low, so lane 0's low word comes first
  const uint32_t kk = st.cursor + 2u * (31u - (uint32_t)lane);
  st_global(end - 1 - kk, (Word)(st.x >> F::kWordBits));
  st_global(end - 2 - kk, (Word)st.x);
  if (lane == 0) c.lens[s] = sizeof(Word) * (uint64_t)(st.cursor + 64);
}

template <class F, typename SymT, bool IB0, bool FLT, bool ST>
__device__ __forceinline__ void encode_stream_w32_entry(const EncCtx &c, const RowMeta *meta,
                                                        const uint32_t *buckets, uint32_t *stg,
                                                        int64_t s, const float *stab) {
  const StreamDesc d = stream_desc(c.g, s);
  if (!d.ok) {
    if ((threadIdx.x & 31) == 0) report(c.status, RANS_ERR_ARG, s);
    return;
  }
  if (d.n == 0) {  // flush the 32 initial states only
    using Word = typename F::Word;
    const int lane = threadIdx.x & 31;
    Word *end = reinterpret_cast<Word *>(c.scratch + slot_end(c.g, d, s));
    end[-1 - 2 * (31 - lane)] = (Word)(F::kLow >> F::kWordBits);
    end[-2 - 2 * (31 - lane)] = (Word)F::kLow;
    if (lane == 0) c.lens[s] = 64 * sizeof(Word);
    return;
  }
  if (d.t.ww >= 32)
    encode_stream_w32<F, SymT, IB0, true, FLT, ST>(c, d, meta, buckets, stg, s, stab);
  else
    encode_stream_w32<F, SymT, IB0, false, FLT, ST>(c, d, meta, buckets, stg, s, stab);
}

template <class F, typename SymT, bool FLT, bool ST>
__device__ void encode_stream_w1(const EncCtx &c, const RowMeta *meta, const uint32_t *buckets,
                                 int64_t s, const float *stab) {
  using Word = typename F::Word;
  const StreamDesc d = stream_desc(c.g, s);
  if (!d.ok) {
    report(c.status, RANS_ERR_ARG, s);
    return;
  }
  Word *end = reinterpret_cast<Word *>(c.scratch + slot_end(c.g, d, s));
  const uint32_t sh = F::shift(c.sh);
  const int ib = c.g.ib_shift;
  const Tile t = d.t;
  const int32_t n = (int32_t)d.n;
  typename F::State x = F::kLow;
  uint32_t cursor = 0;
  RelPos pf, pp;  // next symbol to fetch into the ring; next L2 prefetch
  pf.init(t, n > 0 ? n - 1 : 0);
  pp = pf;
  constexpr int32_t kAhead = 64;
  for (int32_t u = 0; u < kAhead && u < n; ++u) {
    const int64_t p = d.base + pp.rel(t);
    if (FLT) {
      prefetch_l2(c.fy + p);
      prefetch_l2(c.fscale + p);
    } else {
      prefetch_l2(reinterpret_cast<const SymT *>(c.sym) + p);
      prefetch_l2(c.idx + (p >> ib));
    }
    pp.back(t, 1);
  }
  // The symbols and rows of the next kRing symbols (in coding order) wait in
  // registers, each read kRing symbols before it is coded, so that the state
  // chain does not wait on their loads.  FLT: the row and the quantised
  // symbol are computed when read (ok: the value was in range).
  constexpr int kRing = 4;
  int32_t rsym[kRing], rrow[kRing];
  bool rok[kRing];
  auto fetch = [&](int32_t &sv, int32_t &r, bool &ok) {
    const int64_t p = d.base + pf.rel(t);
    pf.back(t, 1);
    ok = true;
    if (FLT) {
      sv = quantize(__ldg(c.fy + p), c.fmean ? __ldg(c.fmean + p) : 0.0f, ok);
      r = (int32_t)scale_row(bound_scale(__ldg(c.fscale + p), c.bound), stab, c.K);
    } else {
      sv = SymIO<SymT>::load(c.sym, p);
      r = __ldg(c.idx + (p >> ib));
    }
  };
#pragma unroll
  for (int u = 0; u < kRing; ++u) {
    rsym[u] = rrow[u] = 0;
    rok[u] = true;
    if (u < n) fetch(rsym[u], rrow[u], rok[u]);
  }
  for (int32_t i = n - 1; i >= 0; --i) {
    const int32_t sv = rsym[0], r = rrow[0];
    const bool ok = rok[0];
#pragma unroll
    for (int u = 0; u + 1 < kRing; ++u) {
      rsym[u] = rsym[u + 1];
      rrow[u] = rrow[u + 1];
      rok[u] = rok[u + 1];
    }
    if (i - kRing >= 0) fetch(rsym[kRing - 1], rrow[kRing - 1], rok[kRing - 1]);
    if (i - kAhead >= 0) {
      const int64_t q = d.base + pp.rel(t);
      if (FLT) {
        prefetch_l2(c.fy + q);
        prefetch_l2(c.fscale + q);
      } else {
        prefetch_l2(reinterpret_cast<const SymT *>(c.sym) + q);
        prefetch_l2(c.idx + (q >> ib));
      }
      pp.back(t, 1);
    }
    if (!ok) {
      report(c.status, RANS_ERR_RANGE, s);
      return;
    }
    if ((uint32_t)r >= (uint32_t)c.K) {
      report(c.status, RANS_ERR_INDEX, s);
      return;
    }
    uint32_t start, freq;
    uint64_t raw;
    bool esc;
    map_symbol<ST>(sv, row_meta(meta, (uint32_t)r), buckets, start, freq, raw, esc);
    if (esc && (raw >> 60) != 0) {
      report(c.status, RANS_ERR_RANGE, s);
      return;
    }
    cursor += symbol_ops<F, true>(x, start, freq, F::rcp(freq, sh), raw, esc, end, cursor, sh);
  }
  end[-1 - (int64_t)cursor] = (Word)(x >> F::kWordBits);
  end[-2 - (int64_t)cursor] = (Word)x;
  cursor += 2;
  c.lens[s] = sizeof(Word) * (uint64_t)cursor;
}

// One state on a contiguous stream (symbol i at base + i), coded last to
// first four symbols a step: the step's symbols and rows are read a step
// ahead, and its four buckets, reciprocals and escapes are looked up before
// the first state update (they do not depend on the state); the symbol
// step is encode_stream_w1's.
template <class F, typename SymT, bool ST>
__device__ void encode_stream_w1c(const EncCtx &c, const RowMeta *meta, const uint32_t *buckets,
                                  int64_t s) {
  using Word = typename F::Word;
  const StreamDesc d = stream_desc(c.g, s);
  if (!d.ok) {
    report(c.status, RANS_ERR_ARG, s);
    return;
  }
  Word *end = reinterpret_cast<Word *>(c.scratch + slot_end(c.g, d, s));
  const uint32_t sh = F::shift(c.sh);
  const int ib = c.g.ib_shift;
  const int32_t n = (int32_t)d.n;
  const int64_t base = d.base;
  const uint32_t kmax = (uint32_t)c.K - 1u;
  typename F::State x = F::kLow;
  uint32_t cursor = 0;
  // the step that codes j, j - 1, j - 2, j - 3
  auto load4 = [&](int32_t j, int32_t (&sv)[4], int32_t (&r)[4]) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int32_t p = j - u;
      sv[u] = p >= 0 ? SymIO<SymT>::load(c.sym, base + p) : 0;
      r[u] = p >= 0 ? __ldg(c.idx + ((base + p) >> ib)) : 0;
    }
  };
  auto prefetch_at = [&](int32_t p) {
    prefetch_l2(reinterpret_cast<const SymT *>(c.sym) + base + p);
    prefetch_l2(c.idx + ((base + p) >> ib));
  };
  for (int32_t q = n - 1; q >= 0 && q >= n - 64; q -= 16) prefetch_at(q);
  int32_t sa[4], ra[4], sn[4], rn[4];
  load4(n - 1, sa, ra);
  load4(n - 5, sn, rn);
#pragma unroll 1
  for (int32_t j = n - 1; j >= 0; j -= 4) {
    uint32_t st4[4], fr4[4];
    uint64_t raw4[4];
    bool esc4[4];
    double rcp4[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      map_symbol<ST>(sa[u], row_meta(meta, min((uint32_t)ra[u], kmax)), buckets, st4[u], fr4[u],
                     raw4[u], esc4[u]);
      rcp4[u] = F::rcp(fr4[u], sh);
    }
    if (((n - 1 - j) & 15) == 0 && j - 64 >= 0) prefetch_at(j - 64);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (j - u < 0) break;
      if ((uint32_t)ra[u] >= (uint32_t)c.K) {
        report(c.status, RANS_ERR_INDEX, s);
        return;
      }
      if (esc4[u] && (raw4[u] >> 60) != 0) {
        report(c.status, RANS_ERR_RANGE, s);
        return;
      }
      cursor +=
          symbol_ops<F, true>(x, st4[u], fr4[u], rcp4[u], raw4[u], esc4[u], end, cursor, sh);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      sa[u] = sn[u];
      ra[u] = rn[u];
    }
    load4(j - 8, sn, rn);
  }
  end[-1 - (int64_t)cursor] = (Word)(x >> F::kWordBits);
  end[-2 - (int64_t)cursor] = (Word)x;
  cursor += 2;
  c.lens[s] = sizeof(Word) * (uint64_t)cursor;
}

// W = 2, 4 or 8 interleaved states on W consecutive lanes of a warp, 32 / W
// streams per warp (the sub-warp groups of "torch_ans 0.3.0", Usage legend).
// Lane l of a segment holds state l and codes symbols l, l + W, ... in
// reverse group order; within a group lane W-1 codes first, so lane l's
// words land below those of the segment's lanes > l (ballot + popc within
// the segment); a group holding an escape counts each lane's words and
// places them by a suffix sum over the segment.  The flush pushes lanes
// W-1 .. 0, high word first.  All lanes run the warp's longest stream's
// group count, idle lanes masked.
// ALIAS: alias-coded streams (the symbol op codes on the remapped position).
template <class F, typename SymT, bool ST, bool ALIAS>
__device__ void encode_segment(const EncCtx &c, const RowMeta *meta, const uint32_t *buckets,
                               int64_t s, int W) {
  using Word = typename F::Word;
  using State = typename F::State;
  const int lane = threadIdx.x & 31;
  const int l = lane & (W - 1);
  const int seg0 = lane - l;
  const uint32_t segmask = ((1u << W) - 1u) << seg0;
  const uint32_t above = segmask & (0xfffffffeu << lane);  // the segment's lanes > l
  const uint32_t sh = F::shift(c.sh);
  StreamDesc d;
  d.ok = false;
  d.n = 0;
  d.base = 0;
  d.t = Tile{1, kNoWrap, 0, 0};
  bool live = false;
  if (s >= 0) {
    d = stream_desc(c.g, s);
    live = d.ok;
    if (!live && l == 0) report(c.status, RANS_ERR_ARG, s);
  }
  Word *end = live ? reinterpret_cast<Word *>(c.scratch + slot_end(c.g, d, s)) : nullptr;
  const int32_t n = live ? (int32_t)d.n : 0;
  const int32_t G = (n + W - 1) / W;
  const int32_t Gmax = (int32_t)__reduce_max_sync(kFull, (uint32_t)G);
  const int ib = c.g.ib_shift;
  const uint32_t kmax = (uint32_t)c.K - 1u;
  State x = F::kLow;
  uint32_t cursor = 0;
  bool bad_index = false, bad_range = false;
  auto pos_of = [&](int32_t k) -> int64_t {
    RelPos rp;
    rp.init(d.t, k * W + l);
    return d.base + rp.rel(d.t);
  };
  // this lane's symbol and row index of group k, read one group ahead
  int32_t sn = 0, rn = 0;
  auto load = [&](int32_t k) {
    sn = 0;
    rn = 0;
    if (k >= 0 && k * W + l < n) {
      const int64_t p = pos_of(k);
      sn = SymIO<SymT>::load(c.sym, p);
      rn = __ldg(c.idx + (p >> ib));
    }
  };
  load(Gmax - 1);
  for (int32_t k = Gmax - 1; k >= 0; --k) {
    const bool active = k * W + l < n;
    const int32_t sv = sn;
    const uint32_t r = (uint32_t)rn;
    load(k - 1);
    bad_index |= active && r > kmax;
    uint32_t start, freq;
    uint64_t raw;
    bool esc;
    map_symbol<ST>(sv, row_meta(meta, active && r <= kmax ? r : 0u), buckets, start, freq, raw,
                   esc);
    esc = esc && active;
    bad_range |= esc && (raw >> 60) != 0;
    raw &= (1ull << 60) - 1;
    const double rcp = F::rcp(freq, sh);
    const uint16_t *remap_row =
        ALIAS ? c.remap + ((size_t)(active && r <= kmax ? r : 0u) << (kPrec - sh)) : nullptr;
    if (!__any_sync(kFull, esc)) {
      const bool need = active && F::need_word(x, freq);
      const uint32_t bm = __ballot_sync(kFull, need);
      if (need) st_global(end - 1 - (cursor + __popc(bm & above)), (Word)x);
      if (need) x >>= F::kWordBits;
      cursor += __popc(bm & segmask);
      if (active) {
        if constexpr (ALIAS) x = F::alias_step(x, start, freq, rcp, sh, remap_row);
        else x = F::sym_step(x, start, freq, rcp, sh);
      }
    } else {
      // every lane counts its words, a suffix sum over the segment places them
      uint32_t kw = 0;
      if (active) {
        State y = x;
        kw = symbol_ops<F, false, ALIAS>(y, start, freq, rcp, raw, esc, end, 0, sh, remap_row);
      }
      uint32_t inc = kw;
      for (int o = 1; o < W; o <<= 1) {
        const uint32_t t = __shfl_down_sync(kFull, inc, o);
        if (l + o < W) inc += t;
      }
      const uint32_t total = __shfl_sync(kFull, inc, seg0);
      if (active)
        symbol_ops<F, true, ALIAS>(x, start, freq, rcp, raw, esc, end, cursor + inc - kw, sh,
                                   remap_row);
      cursor += total;
    }
  }
  const uint32_t idx_fails = __ballot_sync(kFull, bad_index) & segmask;
  const uint32_t rng_fails = __ballot_sync(kFull, bad_range) & segmask;
  if (!live) return;
  if (idx_fails || rng_fails) {
    if (l == 0) report(c.status, idx_fails ? RANS_ERR_INDEX : RANS_ERR_RANGE, s);
    return;
  }
  const uint32_t kk = cursor + 2u * (uint32_t)(W - 1 - l);
  st_global(end - 1 - kk, (Word)(x >> F::kWordBits));
  st_global(end - 2 - kk, (Word)x);
  if (l == 0) c.lens[s] = sizeof(Word) * (uint64_t)(cursor + 2 * W);
}

// Shared-memory bytes of a table mode: 0 reads the tables from global
// memory, 1 stages the row metadata and bucket words, 2 the row metadata
// and the 16-bit starts.
__host__ __device__ inline uint32_t enc_table_bytes(int mode, const EncCtx &c) {
  return mode == 1 ? c.meta_bytes + c.bucket_bytes
                   : (mode == 2 ? c.meta_bytes + c.start_bytes : 0u);
}

// ---------------------------------------------- W = 32, tile-staged input --
// Tiled streams whose tile rows are whole 16-byte units go through a leaner
// warp encoder: the row indexes and symbols of 4 tile rows of one channel (a
// chunk of ww / 8 groups) arrive in a per-warp shared-memory ring with two
// tensor-tile copies on one mbarrier, the stream's chunks taken last to
// first (the coder runs backwards).  Stream group g sits in ring slot
// g mod 2 Gc; chunk c fills slots [(c mod 2) Gc, (c mod 2) Gc + Gc).  While
// one chunk codes, the chunk before it lands in the other half, and the one
// two before that is prefetched into L2.  As in the general coder, a group's
// row index is read three groups ahead, its symbol and row metadata two
// ahead and its bucket word and reciprocal one ahead of its state update.
constexpr uint32_t kEncTileRingBytes = 4096;  // 16 groups of indexes + 16 of symbols
constexpr uint32_t kEncTileWaitTries = 1u << 22;

struct EncTileMaps {
  CUtensorMap idx[2];  // row indexes: box (tile width, 4, 1); [1]: last tile column
  CUtensorMap sym[2];  // int32 symbols, same boxes
};

template <class F, bool ST>
__device__ __forceinline__ bool encode_tile_stream(const EncCtx &c, const EncTileMaps &maps,
                                                   const RowMeta *meta, const uint32_t *buckets,
                                                   uint32_t ring, const uint32_t *ring_p,
                                                   uint32_t bar0, uint32_t &par, int64_t s) {
  using Word = typename F::Word;
  const int lane = threadIdx.x & 31;
  const Geom &g = c.g;
  const StreamDesc d = stream_desc(g, s);
  if (!d.ok) {
    if (lane == 0) report(c.status, RANS_ERR_ARG, s);
    return true;
  }
  Word *end = reinterpret_cast<Word *>(c.scratch + slot_end(g, d, s));
  const uint32_t sh = F::shift(c.sh);
  const uint32_t kmax = (uint32_t)c.K - 1u;
  const uint32_t above = 0xfffffffeu << lane;  // lanes > this lane
  // the tile: image b, channel group gi, tile row ty, tile column tx
  const int64_t per_img = g.ng * g.nty * g.ntx;
  const int64_t b = s / per_img, t0 = s - b * per_img;
  const int64_t gi = t0 / (g.nty * g.ntx), t1 = t0 - gi * (g.nty * g.ntx);
  const int64_t ty = t1 / g.ntx, tx = t1 - ty * g.ntx;
  const int32_t x0 = (int32_t)(tx * g.tw);
  const int32_t ww = d.t.ww, hh = d.t.hh;
  const int cls = ww == (int32_t)g.tw ? 0 : 1;
  const void *imap = &maps.idx[cls];
  const void *smap = &maps.sym[cls];
  const int32_t Gc = ww >> 3;                    // groups per chunk (>= 4)
  const int32_t M = (int32_t)(d.n / (4 * ww));   // chunks
  const int32_t G = M * Gc;
  const uint32_t cbytes = 16u * (uint32_t)ww;
  const uint32_t half = (uint32_t)Gc * 128u;     // bytes of one half of either ring
  const uint32_t sym_w = kEncTileRingBytes / 8;  // word offset of the symbol ring
  // tensor-tile coordinates of chunks, stepped back 4 rows at a time from the
  // last chunk: ld for the loads into shared memory, pf for the L2 prefetches
  struct Back {
    int32_t y, z, y0, ylast;
    __device__ __forceinline__ void prev() {
      y -= 4;
      if (y < y0) {
        y = ylast;
        --z;
      }
    }
  };
  Back ld;
  ld.y0 = (int32_t)(ty * g.th);
  ld.ylast = ld.y = ld.y0 + hh - 4;
  ld.z = (int32_t)(b * g.C + gi * g.cg) + (int32_t)(d.n / ((int64_t)hh * ww)) - 1;
  Back pf = ld;
  const uint32_t bar1 = bar0 + 8;
  uint32_t pending = 0;  // loads in flight, by half
  // the load of stream chunk ch (into half ch & 1); chunks are loaded in
  // descending order
  auto issue = [&](int32_t ch) {
    const int h = ch & 1;
    if (lane == 0) {
      const uint32_t bar = h ? bar1 : bar0;
      tma::fence_proxy_async();
      tma::arrive_expect(bar, 2u * cbytes);
      tma::load_3d(ring + (uint32_t)h * half, imap, x0, ld.y, ld.z, bar);
      tma::load_3d(ring + 4u * sym_w + (uint32_t)h * half, smap, x0, ld.y, ld.z, bar);
    }
    pending |= 1u << h;
    ld.prev();
  };
  auto prefetch = [&]() {
    if (lane == 0) {
      tma::prefetch_l2_3d(imap, x0, pf.y, pf.z);
      tma::prefetch_l2_3d(smap, x0, pf.y, pf.z);
    }
    pf.prev();
  };
  auto wait_chunk = [&](int32_t ch) -> bool {
    const int h = ch & 1;
    const uint32_t bar = h ? bar1 : bar0;
    const bool ok = tma::wait_bounded(bar, (par >> h) & 1u, kEncTileWaitTries);
    if (__all_sync(kFull, ok)) {
      par ^= 1u << h;
      pending &= ~(1u << h);
      return true;
    }
    if (lane == 0) report(c.status, RANS_ERR_TIMEOUT, s);
    for (int q = 0; q < 2; ++q)
      if (pending >> q & 1u) tma::wait_bounded(q ? bar1 : bar0, (par >> q) & 1u, kEncTileWaitTries);
    return false;
  };
  __syncwarp();
  issue(M - 1);
  if (M > 1) issue(M - 2);
  pf.prev();
  if (M > 1) pf.prev();
  for (int32_t q = 2; q < 4 && q < M; ++q) prefetch();

  WarpEnc<F> st;
  st.x = F::kLow;
  st.cursor = 0;
  st.rmax = 0;
  st.range_err = false;
  auto meta_of = [&](uint32_t r) -> RowMeta {
    st.rmax = max(st.rmax, r);
    return row_meta(meta, min(r, kmax));
  };
  // stream group gg sits in ring slot gg mod 2 Gc
  const int32_t nslot = 2 * Gc;
  auto dn = [&](int32_t sl) { return sl == 0 ? nslot - 1 : sl - 1; };
  if (!wait_chunk(M - 1)) return false;
  // groups G - 1 .. G - 3 are in the last chunk (Gc >= 4)
  const int32_t sl_a = (G - 1) % nslot;
  const int32_t sl_b = dn(sl_a), sl_c = dn(sl_b);
  EncLook L = enc_look<F>(
      enc_bucket<ST>((int32_t)ring_p[sym_w + sl_a * 32 + lane], meta_of(ring_p[sl_a * 32 + lane]),
                     buckets),
      true, sh);
  int32_t s1 = (int32_t)ring_p[sym_w + sl_b * 32 + lane];
  RowMeta m1 = meta_of(ring_p[sl_b * 32 + lane]);
  uint32_t r2 = ring_p[sl_c * 32 + lane];
  // reads ahead: the row index of group g3 = G - 4 - k and the symbol of
  // g2 = G - 3 - k, each with its chunk and place in the chunk and ring slot
  int32_t g3 = G - 4, c3 = g3 >= 0 ? g3 / Gc : -1, j3 = g3 >= 0 ? g3 - c3 * Gc : 0;
  int32_t g2 = G - 3, c2 = g2 / Gc, j2 = g2 - c2 * Gc;
  int32_t sl3 = dn(sl_c), sl2 = sl_c;
#pragma unroll 1
  for (int32_t k = 0; k < G; ++k) {
    // group G - 1 - k codes, G - 2 - k is looked up
    const EncBucket b1 = enc_bucket<ST>(s1, m1, buckets);
    const typename F::State x0 = st.x;
    const uint32_t c0 = st.cursor;
    enc_group_fast<F, true>(st, L, true, above, end, sh);
    const EncLook L1 = enc_look<F>(b1, true, sh);
    uint32_t r3 = 0;
    if (g3 >= 0) {
      if (j3 == Gc - 1 && c3 < M - 1) {  // the first read of chunk c3
        if (!wait_chunk(c3)) return false;
      }
      r3 = ring_p[sl3 * 32 + lane];
    }
    int32_t s2 = 0;
    RowMeta m2 = m1;
    if (g2 >= 0) {
      s2 = (int32_t)ring_p[sym_w + sl2 * 32 + lane];
      m2 = meta_of(r2);
      // the last read of chunk c2: the chunk two before it may land in its
      // half, and one four before it go to L2
      if (j2 == 0 && c2 >= 2) {
        __syncwarp();
        issue(c2 - 2);
        if (c2 >= 4) prefetch();
      }
    }
    if (L.any_esc) enc_group_escape<F>(st, x0, c0, L, true, end, sh);
    L = L1;
    s1 = s2;
    m1 = m2;
    r2 = r3;
    sl3 = dn(sl3);
    sl2 = dn(sl2);
    --g3;
    if (--j3 < 0) {
      j3 = Gc - 1;
      --c3;
    }
    --g2;
    if (--j2 < 0) {
      j2 = Gc - 1;
      --c2;
    }
  }
  if (__any_sync(kFull, st.rmax > kmax)) {
    if (lane == 0) report(c.status, RANS_ERR_INDEX, s);
    return true;
  }
  if (__any_sync(kFull, st.range_err)) {
    if (lane == 0) report(c.status, RANS_ERR_RANGE, s);
    return true;
  }
  // flush: lanes 31..0 push high then low, so lane 0's low word comes first
  const uint32_t kk = st.cursor + 2u * (31u - (uint32_t)lane);
  st_global(end - 1 - kk, (Word)(st.x >> F::kWordBits));
  st_global(end - 2 - kk, (Word)st.x);
  if (lane == 0) c.lens[s] = sizeof(Word) * (uint64_t)(st.cursor + 64);
  return true;
}

// ------------------------------------------ unrolled chunks, no branches --
// The coders' time per group follows their instruction count and the
// branches that cut a group into small blocks.  For 56- and 64-wide tiles (7
// and 8 groups per chunk) a chunk is coded as one unrolled block: the
// compiler is free to run the later groups' lookups (row metadata, bucket
// word, reciprocal) under the earlier groups' state updates, the copy-engine
// work is predicated on lane 0, and escapes are only recorded.  A chunk in
// which a lane met an escape is coded again from its saved state and cursor
// with the escape path; the fast pass before it writes at most one word per
// lane and group, inside the stream's worst-case scratch slot, and the redo
// writes every word the stream keeps.
// FLT: the tiles hold float latents: the index tile is the scales (each
// group's row is its scale's table row, from the scale table `stab` in
// shared memory) and the symbol tile y, coded as rint(y - mean) with the
// means read from global memory at the chunk's start (an out-of-range value
// is recorded and coded as 0).
// FM: 0 int32 rows and symbols, 1 float latents with the scale table
// searched, 2 float latents with its rows read through `keys`.
template <class F, bool ST, int GC, int FM>
__device__ __forceinline__ bool encode_tile_stream_fast(const EncCtx &c, const EncTileMaps &maps,
                                                        const RowMeta *meta,
                                                        const uint32_t *buckets, uint32_t ring,
                                                        const uint32_t *ring_p, uint32_t bar0,
                                                        uint32_t &par, int64_t s,
                                                        const float *stab, const ScaleKeys &keys) {
  constexpr bool FLT = FM != 0;
  using Word = typename F::Word;
  const int lane = threadIdx.x & 31;
  const Geom &g = c.g;
  const StreamDesc d = stream_desc(g, s);
  if (!d.ok) {
    if (lane == 0) report(c.status, RANS_ERR_ARG, s);
    return true;
  }
  Word *end = reinterpret_cast<Word *>(c.scratch + slot_end(g, d, s));
  const uint32_t sh = F::shift(c.sh);
  const uint32_t kmax = (uint32_t)c.K - 1u;
  const uint32_t above = 0xfffffffeu << lane;  // lanes > this lane
  const int64_t per_img = g.ng * g.nty * g.ntx;
  const int64_t b = s / per_img, t0 = s - b * per_img;
  const int64_t gi = t0 / (g.nty * g.ntx), t1 = t0 - gi * (g.nty * g.ntx);
  const int64_t ty = t1 / g.ntx, tx = t1 - ty * g.ntx;
  const int32_t x0 = (int32_t)(tx * g.tw);
  const int32_t hh = d.t.hh;
  const int cls = d.t.ww == (int32_t)g.tw ? 0 : 1;
  const void *imap = &maps.idx[cls];
  const void *smap = &maps.sym[cls];
  const int32_t M = (int32_t)(d.n / (32 * GC));
  const uint32_t cbytes = 128u * GC;
  constexpr uint32_t kHalf = 128u * GC;
  constexpr int kSymW = (int)(kEncTileRingBytes / 8);  // word offset of the symbol ring
  // chunk coordinates stepped back 4 rows at a time from the last chunk: ld
  // for the loads into shared memory, pf for the L2 prefetches
  const int32_t y0 = (int32_t)(ty * g.th), ylast = y0 + hh - 4;
  const int32_t zlast =
      (int32_t)(b * g.C + gi * g.cg) + (int32_t)(d.n / ((int64_t)hh * d.t.ww)) - 1;
  int32_t ly = ylast, lz = zlast;
  int32_t py = ly, pz = lz;
  auto back_if = [&](int32_t &y, int32_t &z, bool on) {
    const int32_t yy = y - 4;
    const bool wrap = yy < y0;
    y = on ? (wrap ? ylast : yy) : y;
    z -= on && wrap ? 1 : 0;
  };
  const uint32_t bar1 = bar0 + 8;
  const uint32_t l0 = lane == 0 ? 1u : 0u;
  uint32_t pending = 0;
  // the load of stream chunk ch into half ch & 1 (chunks load in descending order)
  auto issue_if = [&](int32_t ch, uint32_t on) {
    const int h = ch & 1;
    const uint32_t bar = h ? bar1 : bar0;
    tma::fence_proxy_async();
    tma::arrive_expect_if(l0 & on, bar, 2u * cbytes);
    tma::load_3d_if(l0 & on, ring + (uint32_t)h * kHalf, imap, x0, ly, lz, bar);
    tma::load_3d_if(l0 & on, ring + 4u * kSymW + (uint32_t)h * kHalf, smap, x0, ly, lz, bar);
    pending |= on << h;
    back_if(ly, lz, on != 0);
  };
  auto prefetch_if = [&](uint32_t on) {
    tma::prefetch_l2_3d_if(l0 & on, imap, x0, py, pz);
    tma::prefetch_l2_3d_if(l0 & on, smap, x0, py, pz);
    back_if(py, pz, on != 0);
  };
  auto wait_chunk = [&](int32_t ch) -> bool {
    const int h = ch & 1;
    const uint32_t bar = h ? bar1 : bar0;
    const bool ok = tma::wait_bounded(bar, (par >> h) & 1u, kEncTileWaitTries);
    if (__all_sync(kFull, ok)) {
      par ^= 1u << h;
      pending &= ~(1u << h);
      return true;
    }
    if (lane == 0) report(c.status, RANS_ERR_TIMEOUT, s);
    for (int q = 0; q < 2; ++q)
      if (pending >> q & 1u) tma::wait_bounded(q ? bar1 : bar0, (par >> q) & 1u, kEncTileWaitTries);
    return false;
  };
  __syncwarp();
  issue_if(M - 1, 1u);
  back_if(py, pz, true);
  for (int32_t q = 1; q < 3; ++q) prefetch_if(M - 1 - q >= 0 ? 1u : 0u);

  WarpEnc<F> st;
  st.x = F::kLow;
  st.cursor = 0;
  st.rmax = 0;
  st.range_err = false;
  auto meta_of = [&](uint32_t r) -> RowMeta {
    if (FM == 1) r = scale_row(bound_scale(__uint_as_float(r), c.bound), stab, c.K);
    if (FM == 2) r = keys.row(bound_scale(__uint_as_float(r), c.bound));
    st.rmax = max(st.rmax, r);
    return row_meta(meta, min(r, kmax));
  };
  // FLT: the chunk's means (0 without means), read one chunk ahead (my, mz:
  // the next chunk's position), and the symbol of a staged y.  Group j's
  // lane reads element e = 32 j + lane of the chunk: row e / ww, column
  // e mod ww.
  float mu[GC], mu_n[GC];
#pragma unroll
  for (int j = 0; j < GC; ++j) mu[j] = mu_n[j] = 0.0f;
  int32_t moff[GC];
  int32_t my = ylast, mz = zlast;  // the last chunk's position
  if (FLT) {
#pragma unroll
    for (int j = 0; j < GC; ++j) {
      const int e = j * 32 + lane, r = e / (8 * GC);
      moff[j] = r * (int32_t)g.Wd + (e - r * 8 * GC);
    }
  }
  auto load_means = [&](bool on, float (&m)[GC]) {
#pragma unroll
    for (int j = 0; j < GC; ++j) m[j] = 0.0f;
    if (c.fmean && on) {
      const float *mp = c.fmean + (((int64_t)mz * g.H + my) * g.Wd + x0);
#pragma unroll
      for (int j = 0; j < GC; ++j) m[j] = __ldg(mp + moff[j]);
    }
    back_if(my, mz, on);
  };
  if (FLT) load_means(true, mu_n);
  auto sym_of = [&](uint32_t v, float mean) -> int32_t {
    if (!FLT) return (int32_t)v;
    bool ok;
    const int32_t q = quantize(__uint_as_float(v), mean, ok);
    st.range_err |= !ok;
    return q;
  };
#pragma unroll 1
  for (int32_t ch = M - 1; ch >= 0; --ch) {
    if (FLT) {
#pragma unroll
      for (int j = 0; j < GC; ++j) mu[j] = mu_n[j];
      load_means(ch >= 1, mu_n);
    }
    if (!wait_chunk(ch)) return false;
    // the chunk before this one into the other half (consumed by the chunk
    // after this one), and the one three before it into L2
    __syncwarp();
    issue_if(ch - 1, ch >= 1 ? 1u : 0u);
    prefetch_if(ch >= 3 ? 1u : 0u);
    const uint32_t *ri = ring_p + (ch & 1) * (int)(kHalf / 4);
    const uint32_t *rs = ri + kSymW;
    const typename F::State xs = st.x;
    const uint32_t cs = st.cursor;
    uint32_t esc = 0;
    // every group's bucket first, since the lookups do not depend on the
    // state
    uint32_t be[GC];
#pragma unroll
    for (int j = GC - 1; j >= 0; --j) {
      const EncBucket bk = enc_bucket<ST>(sym_of(rs[j * 32 + lane], mu[j]),
                                          meta_of(ri[j * 32 + lane]), buckets);
      esc |= bk.in_range ? 0u : 1u;
      be[j] = bk.e;
    }
#pragma unroll
    for (int j = GC - 1; j >= 0; --j) {
      EncLook L;
      L.start = bucket_start(be[j]);
      L.freq = bucket_freq(be[j]);
      L.rcp = F::rcp(L.freq, sh);
      enc_group_fast<F, true>(st, L, true, above, end, sh);
    }
    if (__any_sync(kFull, esc != 0)) {
      // an escape in this chunk: code it again from its saved state
      st.x = xs;
      st.cursor = cs;
#pragma unroll 1
      for (int j = GC - 1; j >= 0; --j) {
        float mj = 0.0f;
#pragma unroll
        for (int q = 0; q < GC; ++q) mj = q == j ? mu[q] : mj;
        const EncBucket bk = enc_bucket<ST>(sym_of(rs[j * 32 + lane], mj),
                                            meta_of(ri[j * 32 + lane]), buckets);
        const EncLook L = enc_look<F>(bk, true, sh);
        const typename F::State xg = st.x;
        const uint32_t cg = st.cursor;
        enc_group_fast<F, true>(st, L, true, above, end, sh);
        if (L.any_esc) enc_group_escape<F>(st, xg, cg, L, true, end, sh);
      }
    }
  }
  if (__any_sync(kFull, st.rmax > kmax)) {
    if (lane == 0) report(c.status, RANS_ERR_INDEX, s);
    return true;
  }
  if (__any_sync(kFull, st.range_err)) {
    if (lane == 0) report(c.status, RANS_ERR_RANGE, s);
    return true;
  }
  const uint32_t kk = st.cursor + 2u * (31u - (uint32_t)lane);
  st_global(end - 1 - kk, (Word)(st.x >> F::kWordBits));
  st_global(end - 2 - kk, (Word)st.x);
  if (lane == 0) c.lens[s] = sizeof(Word) * (uint64_t)(st.cursor + 64);
  return true;
}

// Float latents: at most 16 warps a CTA, so that the extra per-element work
// (the row and the symbol of each scale and y) has registers to spare.
constexpr int kEncFltMaxWarps = 16;

template <class F, bool ST, bool FLT>
__global__ void __launch_bounds__(FLT ? kEncFltMaxWarps * 32 : kEncThreads32, 1)
    encode_tile_kernel(EncCtx c, const __grid_constant__ EncTileMaps maps) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ uint64_t bar;
  __shared__ uint64_t ring_bar[kEncMaxWarps][2];
  const char *gb = c.blob + kHeaderBytes;
  if (ST) {
    if (!stage_to_smem(smem, gb, c.meta_bytes, &bar, c.status, smem + c.meta_bytes,
                       gb + c.meta_bytes + c.bucket_bytes, c.start_bytes))
      return;
  } else {
    if (!stage_to_smem(smem, gb, c.meta_bytes + c.bucket_bytes, &bar, c.status)) return;
  }
  const RowMeta *meta = reinterpret_cast<const RowMeta *>(smem);
  const uint32_t *buckets = reinterpret_cast<const uint32_t *>(smem + c.meta_bytes);
  const uint32_t tab = enc_table_bytes(ST ? 2 : 1, c);
  const int warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5, lane = threadIdx.x & 31;
  const uint32_t sbase = smem_addr(smem);
  const uint32_t ring = ((sbase + tab + 127u) & ~127u) + (uint32_t)warp * kEncTileRingBytes;
  const uint32_t *ring_p = reinterpret_cast<const uint32_t *>(smem + (ring - sbase));
  const uint32_t bar0 = smem_addr(&ring_bar[warp][0]);
  // FLT: the scale table after every warp's ring, then its key counts
  float *stab = nullptr;
  ScaleKeys keys{};
  bool use_keys = false;
  if (FLT) {
    stab = reinterpret_cast<float *>(smem + (((sbase + tab + 127u) & ~127u) - sbase) +
                                     (uint32_t)nwarp * kEncTileRingBytes);
    for (int i = threadIdx.x; i < c.K; i += blockDim.x) stab[i] = c.stab[i];
    __syncthreads();
    use_keys = build_scale_keys(
        stab, c.K, c.bound,
        reinterpret_cast<uint16_t *>(reinterpret_cast<char *>(stab) + pad16(4ull * c.K)), keys);
  }
  if (lane == 0) {
    tma::mbar_init(bar0, 1);
    tma::mbar_init(bar0 + 8, 1);
    tma::fence_mbar_init();
  }
  __syncwarp();
  uint32_t par = 0;
  for (int64_t k = blockIdx.x + (int64_t)gridDim.x * warp; k < c.g.S;
       k += (int64_t)gridDim.x * nwarp) {
    const int64_t s = stream_of(c.g, k);
    // unrolled chunks for tile widths 64 and 56 (8 and 7 groups), the general
    // loop otherwise (float latents take the tile kernel only when every tile
    // is 64 or 56 wide)
    const int64_t ww = c.g.tw * ((s % c.g.ntx) + 1) <= c.g.Wd ? c.g.tw : c.g.Wd % c.g.tw;
    bool ok = true;
    switch (ww) {
      case 64:
        if (FLT && use_keys)
          ok = encode_tile_stream_fast<F, ST, 8, 2>(c, maps, meta, buckets, ring, ring_p, bar0, par, s, stab, keys);
        else
          ok = encode_tile_stream_fast<F, ST, 8, FLT ? 1 : 0>(c, maps, meta, buckets, ring, ring_p, bar0, par, s, stab, keys);
        break;
      case 56:
        if (FLT && use_keys)
          ok = encode_tile_stream_fast<F, ST, 7, 2>(c, maps, meta, buckets, ring, ring_p, bar0, par, s, stab, keys);
        else
          ok = encode_tile_stream_fast<F, ST, 7, FLT ? 1 : 0>(c, maps, meta, buckets, ring, ring_p, bar0, par, s, stab, keys);
        break;
      default:
        if constexpr (FLT) {
          if (lane == 0) report(c.status, RANS_ERR_ARG, s);
        } else {
          ok = encode_tile_stream<F, ST>(c, maps, meta, buckets, ring, ring_p, bar0, par, s);
        }
    }
    if (!ok) break;
  }
}

// --------------------------------------------- contiguous chunked streams --
// Contiguous streams (64-bit format, W = 32) made of whole chunks of 256
// symbols whose row changes at most once per chunk (an index block of 256
// symbols or more; the byte sweep's shape): a chunk's row index is one load,
// read a chunk ahead, and its row metadata one shared load; its symbols come
// into a two-half ring in shared memory with 16-byte cp.async copies, a
// chunk ahead; its 8 groups are coded as one unrolled block (escapes only
// recorded, the chunk coded again from its saved state when one occurs), in
// the same order as the general coder, so the streams are the same.
constexpr int kEncChunkSyms = 256;

// PER: one row index per symbol, copied with the symbols into an index
// ring (else one per chunk, read directly).  RCP: rtab holds every bucket's
// divisor reciprocal (F::rcp of its width, the same double), read beside
// its bucket word instead of computed per group.
template <typename SymT, bool ST, bool PER, bool RCP = false>
__device__ __forceinline__ void encode_chunk_stream(const EncCtx &c, const RowMeta *meta,
                                                    const uint32_t *buckets, SymT *ring,
                                                    int32_t *iring, int64_t s,
                                                    const double *rtab = nullptr) {
  using F = Rans64;
  using Word = typename F::Word;
  constexpr int GC = kEncChunkSyms / 32;
  constexpr int kChunkBytes = kEncChunkSyms * (int)sizeof(SymT);
  const int lane = threadIdx.x & 31;
  const Geom &g = c.g;
  const StreamDesc d = stream_desc(g, s);
  if (!d.ok) {
    if (lane == 0) report(c.status, RANS_ERR_ARG, s);
    return;
  }
  Word *end = reinterpret_cast<Word *>(c.scratch + slot_end(g, d, s));
  const uint32_t sh = 0;
  const uint32_t kmax = (uint32_t)c.K - 1u;
  const uint32_t above = 0xfffffffeu << lane;  // lanes > this lane
  const SymT *src = reinterpret_cast<const SymT *>(c.sym) + d.base;
  const int32_t M = (int32_t)(d.n / kEncChunkSyms);
  const int ib = g.ib_shift;
  // chunk ch's symbols (PER: and rows) into ring half ch & 1 (one commit
  // group per call)
  auto issue = [&](int32_t ch) {
    const char *gs = reinterpret_cast<const char *>(src + (int64_t)ch * kEncChunkSyms);
    char *ds = reinterpret_cast<char *>(ring + (ch & 1) * kEncChunkSyms);
#pragma unroll
    for (int o = lane * 16; o < kChunkBytes; o += 32 * 16) cp_async16(ds + o, gs + o);
    if (PER) {
      const int32_t *gi = c.idx + d.base + (int64_t)ch * kEncChunkSyms;
      int32_t *di = iring + (ch & 1) * kEncChunkSyms;
#pragma unroll
      for (int o = lane * 4; o < kEncChunkSyms; o += 128) cp_async16(di + o, gi + o);
    }
    cp_async_commit();
  };
  auto row_at = [&](int32_t ch) -> uint32_t {
    return PER ? 0u : (uint32_t)__ldg(c.idx + ((d.base + (int64_t)ch * kEncChunkSyms) >> ib));
  };
  WarpEnc<F> st;
  st.x = F::kLow;
  st.cursor = 0;
  st.rmax = 0;
  st.range_err = false;
  issue(M - 1);
  uint32_t r_next = row_at(M - 1);
#pragma unroll 1
  for (int32_t ch = M - 1; ch >= 0; --ch) {
    const uint32_t r = r_next;
    // the chunk before this one into the other half (read two chunks ago),
    // then this chunk's symbols landed
    __syncwarp();
    if (ch >= 1) {
      issue(ch - 1);
      r_next = row_at(ch - 1);
    } else {
      cp_async_commit();
    }
    cp_async_wait<1>();
    __syncwarp();
    const SymT *rs = ring + (ch & 1) * kEncChunkSyms;
    const int32_t *ri = iring + (ch & 1) * kEncChunkSyms;
    // group j's row metadata: the chunk's, or (PER) each lane's own
    auto meta_j = [&](int j) -> RowMeta {
      const uint32_t rj = PER ? (uint32_t)ri[j * 32 + lane] : r;
      st.rmax = max(st.rmax, rj);
      return row_meta(meta, min(rj, kmax));
    };
    const typename F::State xs = st.x;
    const uint32_t cs = st.cursor;
    uint32_t esc = 0;
    uint32_t be[GC];  // bucket words, or (RCP) bucket indexes
#pragma unroll
    for (int j = GC - 1; j >= 0; --j) {
      if constexpr (RCP) {
        const RowMeta m = meta_j(j);
        const int64_t v = (int64_t)rs[j * 32 + lane] - (int64_t)m.offset;
        const bool in = (uint64_t)v < (uint64_t)m.maxv;
        esc |= in ? 0u : 1u;
        be[j] = m.bucket_base + (in ? (uint32_t)v : m.maxv);
      } else {
        const EncBucket bk = enc_bucket<ST>((int32_t)rs[j * 32 + lane], meta_j(j), buckets);
        esc |= bk.in_range ? 0u : 1u;
        be[j] = bk.e;
      }
    }
#pragma unroll
    for (int j = GC - 1; j >= 0; --j) {
      EncLook L;
      const uint32_t e = RCP ? buckets[be[j]] : be[j];
      L.start = bucket_start(e);
      L.freq = bucket_freq(e);
      L.rcp = RCP ? rtab[be[j]] : F::rcp(L.freq, sh);
      enc_group_fast<F, true>(st, L, true, above, end, sh);
    }
    if (__any_sync(kFull, esc != 0)) {
      // an escape in this chunk: code it again from its saved state
      st.x = xs;
      st.cursor = cs;
#pragma unroll 1
      for (int j = GC - 1; j >= 0; --j) {
        const EncBucket bk = enc_bucket<ST>((int32_t)rs[j * 32 + lane], meta_j(j), buckets);
        const EncLook L = enc_look<F>(bk, true, sh);
        const typename F::State xg = st.x;
        const uint32_t cg = st.cursor;
        enc_group_fast<F, true>(st, L, true, above, end, sh);
        if (L.any_esc) enc_group_escape<F>(st, xg, cg, L, true, end, sh);
      }
    }
  }
  cp_async_wait<0>();
  if (__any_sync(kFull, st.rmax > kmax)) {
    if (lane == 0) report(c.status, RANS_ERR_INDEX, s);
    return;
  }
  if (__any_sync(kFull, st.range_err)) {
    if (lane == 0) report(c.status, RANS_ERR_RANGE, s);
    return;
  }
  // flush: lanes 31..0 push high then low, so lane 0's low word comes first
  const uint32_t kk = st.cursor + 2u * (31u - (uint32_t)lane);
  st_global(end - 1 - kk, (Word)(st.x >> F::kWordBits));
  st_global(end - 2 - kk, (Word)st.x);
  if (lane == 0) c.lens[s] = sizeof(Word) * (uint64_t)(st.cursor + 64);
}

constexpr int kEncChunkMaxWarps = 32;  // a 2^28-symbol sweep's 8,192 streams in two rounds

// Shared memory per warp: the two-half symbol ring, and (PER) the two-half
// index ring.
template <typename SymT, bool PER>
__host__ __device__ constexpr uint32_t enc_chunk_warp_bytes() {
  return 2u * kEncChunkSyms * (uint32_t)sizeof(SymT) + (PER ? 2u * kEncChunkSyms * 4u : 0u);
}

// Bytes of the bucket reciprocal table (RCP): one double per bucket word.
__host__ __device__ inline uint32_t enc_rcp_bytes(const EncCtx &c) {
  return 2u * c.bucket_bytes;
}

template <typename SymT, bool ST, bool PER, bool RCP = false>
__global__ void __launch_bounds__(kEncChunkMaxWarps * 32, 1) encode_chunk_kernel(EncCtx c) {
  static_assert(!RCP || !ST, "reciprocals beside bucket words");
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ uint64_t bar;
  const char *gb = c.blob + kHeaderBytes;
  if (ST) {
    if (!stage_to_smem(smem, gb, c.meta_bytes, &bar, c.status, smem + c.meta_bytes,
                       gb + c.meta_bytes + c.bucket_bytes, c.start_bytes))
      return;
  } else {
    if (!stage_to_smem(smem, gb, c.meta_bytes + c.bucket_bytes, &bar, c.status)) return;
  }
  const RowMeta *meta = reinterpret_cast<const RowMeta *>(smem);
  const uint32_t *buckets = reinterpret_cast<const uint32_t *>(smem + c.meta_bytes);
  uint32_t tab = enc_table_bytes(ST ? 2 : 1, c);
  double *rtab = nullptr;
  if constexpr (RCP) {
    // every bucket's reciprocal, after the tables (16-byte aligned: the
    // tables' sizes are multiples of 16)
    rtab = reinterpret_cast<double *>(smem + tab);
    for (uint32_t j = threadIdx.x; j < c.bucket_bytes / 4u; j += blockDim.x)
      rtab[j] = Rans64::rcp(bucket_freq(buckets[j]), 0u);
    __syncthreads();
    tab += enc_rcp_bytes(c);
  }
  const int warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
  const uint32_t sbase = smem_addr(smem);
  const uint32_t rbase = ((sbase + tab + 127u) & ~127u) + (uint32_t)warp * enc_chunk_warp_bytes<SymT, PER>();
  SymT *ring = reinterpret_cast<SymT *>(smem + (rbase - sbase));
  int32_t *iring = reinterpret_cast<int32_t *>(smem + (rbase - sbase) +
                                               2u * kEncChunkSyms * (uint32_t)sizeof(SymT));
  for (int64_t k = blockIdx.x + (int64_t)gridDim.x * warp; k < c.g.S;
       k += (int64_t)gridDim.x * nwarp)
    encode_chunk_stream<SymT, ST, PER, RCP>(c, meta, buckets, ring, iring, k, rtab);
}

// Whether a tiled W = 32 encode can take the tile-staged kernel (the
// conditions of the decoder's tile path -- int32 rows and symbols in 16-byte
// aligned tensors, one index per element, tile rows of whole 16-byte units
// and 8-symbol steps, tile heights multiples of 4 -- with tile widths of at
// least 32, so that a chunk holds the 4 groups the coder reads ahead) with
// its tables in shared memory.
bool enc_tile_path_ok(const EncCtx &c, int mode, int sym_dtype, const void *indexes,
                      const void *symbols) {
  const Geom &g = c.g;
  if (g.kind != RANS_CHUNK_TILED || g.W != 32 || g.alias || (mode != 1 && mode != 2) ||
      g.ib_shift != 0 || sym_dtype != RANS_SYM_INT32)
    return false;
  if ((reinterpret_cast<uintptr_t>(indexes) & 15) || (reinterpret_cast<uintptr_t>(symbols) & 15))
    return false;
  const int64_t ww1 = g.Wd % g.tw, hh1 = g.H % g.th;
  auto width_ok = [](int64_t w) { return w % 8 == 0 && w >= 32 && w <= 64; };
  if (!width_ok(g.tw > g.Wd ? g.Wd : g.tw) || (ww1 != 0 && !width_ok(ww1))) return false;
  if (g.th % 4 != 0 || hh1 % 4 != 0 || g.Wd % 4 != 0) return false;
  return true;
}

constexpr int kNotTaken = 1;

template <class F, bool FLT = false>
int launch_encode_tile(const EncCtx &c, int mode, const int32_t *indexes, const void *symbols,
                       cudaStream_t st) {
  const Geom &g = c.g;
  int dev = 0;
  cudaGetDevice(&dev);
  const uint32_t tab = enc_table_bytes(mode, c);
  const uint32_t stab_bytes =
      FLT ? (uint32_t)pad16(4ull * (uint64_t)c.K) + kScaleKeyBytes : 0u;
  const int optin = smem_optin(dev);
  const uint32_t lim = (uint32_t)optin - 64u - 2u * 8u * kEncMaxWarps - stab_bytes;
  if (FLT && c.K > 65536) return kNotTaken;
  if (tab + 128u + kEncTileRingBytes > lim) return kNotTaken;
  EncTileMaps maps;
  const int64_t per_img = g.ng * g.nty * g.ntx;
  const int64_t depth = (g.S / per_img) * g.C;
  const uint32_t w0 = (uint32_t)(g.tw > g.Wd ? g.Wd : g.tw);
  const uint32_t w1 = g.Wd % g.tw ? (uint32_t)(g.Wd % g.tw) : w0;
  for (int k = 0; k < 2; ++k) {
    const uint32_t bw = k ? w1 : w0;
    if (encode_tile_map(&maps.idx[k], indexes, g.Wd, g.H, depth, bw, 4) ||
        encode_tile_map(&maps.sym[k], symbols, g.Wd, g.H, depth, bw, 4))
      return RANS_ERR_CUDA;
  }
  const int sms = num_sms(dev);
  int64_t warps = (g.S + sms - 1) / sms;
  const int64_t max_warps = FLT ? kEncFltMaxWarps : kEncMaxWarps;
  if (warps > max_warps) warps = max_warps;
  const int64_t room = ((int64_t)lim - tab - 128) / kEncTileRingBytes;
  if (warps > room) warps = room;
  if (warps < 1) warps = 1;
  const uint32_t smem = tab + 128u + (uint32_t)warps * kEncTileRingBytes + stab_bytes;
  auto kern = mode == 2 ? encode_tile_kernel<F, true, FLT> : encode_tile_kernel<F, false, FLT>;
  if (ensure_dyn_smem((const void *)kern, (uint32_t)(smem)) !=
      cudaSuccess)
    return RANS_ERR_CUDA;
  int fit = 0;
  if (blocks_per_sm(&fit, (const void *)kern, (int)warps * 32, (uint32_t)(smem)) !=
          cudaSuccess ||
      fit < 1)
    return RANS_ERR_CUDA;
  const int64_t need = (g.S + warps - 1) / warps;
  const int64_t cap = (int64_t)fit * sms;
  const int64_t blocks = need < cap ? need : cap;
  kern<<<(unsigned)blocks, (unsigned)warps * 32, smem, st>>>(c, maps);
  return cudaGetLastError() == cudaSuccess ? RANS_OK : RANS_ERR_CUDA;
}

// Whether an encode can take the chunked kernel: contiguous W = 32 streams
// of the 64-bit format, every stream a whole number of 256-symbol chunks, an
// index block of at least 256 symbols, the tables in shared memory, and
// 16-byte aligned 1-, 2- or 4-byte symbols.
bool enc_chunk_path_ok(const EncCtx &c, int mode, int sym_dtype, const void *symbols) {
  const Geom &g = c.g;
  if (g.kind != RANS_CHUNK_CONTIG || g.W != 32 || g.alias || g.fmt != RANS_FMT_RANS64 ||
      (mode != 1 && mode != 2) || (g.ib_shift != 0 && g.ib_shift < 8))
    return false;
  if (g.ib_shift == 0 && (reinterpret_cast<uintptr_t>(c.idx) & 15) != 0) return false;
  if (sym_dtype != RANS_SYM_UINT8 && sym_dtype != RANS_SYM_INT16 && sym_dtype != RANS_SYM_INT32)
    return false;
  if (g.per < kEncChunkSyms || g.per % kEncChunkSyms != 0 || g.n != g.S * g.per) return false;
  return (reinterpret_cast<uintptr_t>(symbols) & 15) == 0;
}

template <typename SymT, bool PER>
int launch_encode_chunk(const EncCtx &c, int mode, cudaStream_t st) {
  const Geom &g = c.g;
  int dev = 0;
  cudaGetDevice(&dev);
  const uint32_t tab = enc_table_bytes(mode, c);
  const uint32_t per_warp = enc_chunk_warp_bytes<SymT, PER>();
  const uint32_t lim = (uint32_t)smem_optin(dev) - 64u;
  if (tab + 128u + per_warp > lim) return kNotTaken;
  const int sms = num_sms(dev);
  int64_t warps = (g.S + sms - 1) / sms;
  if (warps > kEncChunkMaxWarps) warps = kEncChunkMaxWarps;
  // every bucket's reciprocal in shared memory too (chunk rows, bucket
  // words) when it costs no warps and the CTA is wide enough to build it
  // quickly (at most 16 reciprocals a thread)
  const uint32_t rcp = enc_rcp_bytes(c);
  const bool use_rcp = !PER && mode == 1 && tab % 16u == 0 &&
                       (int64_t)tab + rcp + 128 + warps * per_warp <= (int64_t)lim &&
                       (int64_t)(c.bucket_bytes / 4u) <= 16 * 32 * warps;
  const uint32_t tabr = tab + (use_rcp ? rcp : 0u);
  const int64_t room = ((int64_t)lim - tabr - 128) / per_warp;
  if (warps > room) warps = room;
  if (warps < 1) warps = 1;
  const uint32_t smem = tabr + 128u + (uint32_t)warps * per_warp;
  auto kern = mode == 2 ? encode_chunk_kernel<SymT, true, PER>
                        : (use_rcp ? encode_chunk_kernel<SymT, false, PER, !PER>
                                   : encode_chunk_kernel<SymT, false, PER>);
  if (ensure_dyn_smem((const void *)kern, smem) != cudaSuccess) return RANS_ERR_CUDA;
  int fit = 0;
  if (blocks_per_sm(&fit, (const void *)kern, (int)warps * 32, smem) != cudaSuccess || fit < 1)
    return RANS_ERR_CUDA;
  const int64_t need = (g.S + warps - 1) / warps;
  const int64_t cap = (int64_t)fit * sms;
  const int64_t blocks = need < cap ? need : cap;
  kern<<<(unsigned)blocks, (unsigned)warps * 32, smem, st>>>(c);
  return cudaGetLastError() == cudaSuccess ? RANS_OK : RANS_ERR_CUDA;
}

template <class F, int W, typename SymT, int MODE, bool IB0, bool FLT>
__global__ void __launch_bounds__(W == 32 ? kEncThreads32 : kEncThreads1)
    encode_kernel(EncCtx c) {
  constexpr bool ST = MODE == 2;
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ uint64_t bar;
  const RowMeta *meta;
  const uint32_t *buckets;  // bucket words, or (ST) the 16-bit starts
  const char *gb = c.blob + kHeaderBytes;
  if (MODE == 1) {
    if (!stage_to_smem(smem, gb, c.meta_bytes + c.bucket_bytes, &bar, c.status)) return;
    meta = reinterpret_cast<const RowMeta *>(smem);
    buckets = reinterpret_cast<const uint32_t *>(smem + c.meta_bytes);
  } else if (MODE == 2) {
    if (!stage_to_smem(smem, gb, c.meta_bytes, &bar, c.status, smem + c.meta_bytes,
                       gb + c.meta_bytes + c.bucket_bytes, c.start_bytes))
      return;
    meta = reinterpret_cast<const RowMeta *>(smem);
    buckets = reinterpret_cast<const uint32_t *>(smem + c.meta_bytes);
  } else {
    meta = reinterpret_cast<const RowMeta *>(gb);
    buckets = reinterpret_cast<const uint32_t *>(gb + c.meta_bytes);
  }
  const uint32_t tab = enc_table_bytes(MODE, c);
  // FLT: the scale table, copied after the stage rings when it fits
  const float *stab = c.stab;
  if (FLT && c.stab_smem) {
    float *t = reinterpret_cast<float *>(
        smem + tab + (W == 32 ? (blockDim.x >> 5) * enc_stage_bytes_per_warp(FLT) : 0));
    for (int i = threadIdx.x; i < c.K; i += blockDim.x) t[i] = c.stab[i];
    __syncthreads();
    stab = t;
  }
  if (W == 32) {
    const int warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    uint32_t *stg = reinterpret_cast<uint32_t *>(smem + tab) +
                    warp * (enc_stage_bytes_per_warp(FLT) / 4);
    for (int64_t k = blockIdx.x + (int64_t)gridDim.x * warp; k < c.g.S;
         k += (int64_t)gridDim.x * nw)
      encode_stream_w32_entry<F, SymT, IB0, FLT, ST>(c, meta, buckets, stg, stream_of(c.g, k),
                                                     stab);
  } else {
    // contiguous or explicit streams of integer symbols take the four-symbol
    // loop, tiled streams and float latents the general one
    const bool flat = !FLT && c.g.kind != RANS_CHUNK_TILED;
    for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < c.g.S;
         k += (int64_t)gridDim.x * blockDim.x) {
      if constexpr (!FLT) {
        if (flat) {
          encode_stream_w1c<F, SymT, ST>(c, meta, buckets, stream_of(c.g, k));
          continue;
        }
      }
      encode_stream_w1<F, SymT, FLT, ST>(c, meta, buckets, stream_of(c.g, k), stab);
    }
  }
}

// W = 2, 4 or 8: 32 / W streams per warp (encode_segment); the table mode
// (0, 1 or 2 as for encode_kernel) is a run-time argument.
constexpr int kSegThreads = 256;

template <class F, typename SymT, bool ALIAS>
__global__ void __launch_bounds__(kSegThreads) encode_kernel_wn(EncCtx c, int mode) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ uint64_t bar;
  const RowMeta *meta = reinterpret_cast<const RowMeta *>(c.blob + kHeaderBytes);
  const char *gb = c.blob + kHeaderBytes;
  const uint32_t *buckets = reinterpret_cast<const uint32_t *>(gb + c.meta_bytes);
  if (mode == 1) {
    if (!stage_to_smem(smem, gb, c.meta_bytes + c.bucket_bytes, &bar, c.status)) return;
  } else if (mode == 2) {
    if (!stage_to_smem(smem, gb, c.meta_bytes, &bar, c.status, smem + c.meta_bytes,
                       gb + c.meta_bytes + c.bucket_bytes, c.start_bytes))
      return;
  }
  if (mode != 0) {
    meta = reinterpret_cast<const RowMeta *>(smem);
    buckets = reinterpret_cast<const uint32_t *>(smem + c.meta_bytes);
  }
  const int W = c.g.W;
  const int per_warp = 32 / W;
  const int seg = (threadIdx.x & 31) / W;
  const int64_t warp = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t k0 = warp * per_warp; k0 < c.g.S; k0 += nwarps * per_warp) {
    const int64_t k = k0 + seg;
    const int64_t s = k < c.g.S ? stream_of(c.g, k) : -1;
    if (mode == 2)
      encode_segment<F, SymT, true, ALIAS>(c, meta, buckets, s, W);
    else
      encode_segment<F, SymT, false, ALIAS>(c, meta, buckets, s, W);
  }
}

// ---- compaction -----------------------------------------------------------

constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads)
    scan_lengths_kernel(const uint64_t *lens, int64_t S, uint64_t *offsets, uint64_t capacity,
                        int32_t *status) {
  __shared__ unsigned long long warp_tot[kScanThreads / 32];
  __shared__ unsigned long long carry_sh;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    carry_sh = 0;
    offsets[0] = 0;
  }
  __syncthreads();
  for (int64_t base = 0; base < S; base += kScanThreads) {
    const int64_t i = base + threadIdx.x;
    unsigned long long v = i < S ? lens[i] : 0ull;
    unsigned long long inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      unsigned long long t = __shfl_up_sync(kFull, inc, o);
      if (lane >= o) inc += t;
    }
    if (lane == 31) warp_tot[wid] = inc;
    __syncthreads();
    if (wid == 0) {
      unsigned long long w = warp_tot[lane];
      unsigned long long wi = w;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        unsigned long long t = __shfl_up_sync(kFull, wi, o);
        if (lane >= o) wi += t;
      }
      warp_tot[lane] = wi - w;
    }
    __syncthreads();
    const unsigned long long carry = carry_sh;
    const unsigned long long out = carry + warp_tot[wid] + inc;
    if (i < S) offsets[i + 1] = out;
    __syncthreads();
    if (threadIdx.x == kScanThreads - 1) carry_sh = out;
    __syncthreads();
  }
  if (threadIdx.x == 0 && carry_sh > capacity) report(status, RANS_ERR_CAPACITY, -1);
}

// A warp copies `words` words from src to dst with sixteen loads in flight
// per lane.
template <typename Word>
__device__ __forceinline__ void warp_copy_words(Word *dst, const Word *src, uint64_t words) {
  const int lane = threadIdx.x & 31;
  uint64_t k = 0;
  for (; k + 512 <= words; k += 512) {
    Word v[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) v[u] = __ldg(src + k + u * 32 + lane);
#pragma unroll
    for (int u = 0; u < 16; ++u) dst[k + u * 32 + lane] = v[u];
  }
  // the tail: every load first, then every store
  Word v[16];
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    const uint64_t q = k + u * 32 + lane;
    v[u] = q < words ? __ldg(src + q) : Word(0);
  }
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    const uint64_t q = k + u * 32 + lane;
    if (q < words) dst[q] = v[u];
  }
}

// Word: the format's stream word (stream lengths and offsets are multiples
// of its size).
template <typename Word>
__global__ void copy_streams_kernel(Geom g, const char *scratch, const uint64_t *lens,
                                    const uint64_t *offsets, uint8_t *out, uint64_t capacity) {
  const int lane = threadIdx.x & 31;
  const int64_t nw = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t s = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); s < g.S;
       s += nw) {
    const StreamDesc d = stream_desc(g, s);
    if (!d.ok) continue;
    const uint64_t len = lens[s];
    const uint64_t off = offsets[s];
    if (off + len > capacity) continue;
    const Word *src = reinterpret_cast<const Word *>(scratch + slot_end(g, d, s) - len);
    Word *dst = reinterpret_cast<Word *>(out + off);
    const uint64_t words = len / sizeof(Word);
    warp_copy_words(dst, src, words);
  }
}

// Scan and copy in one launch, for up to kFusedMaxStreams streams: block b
// owns streams [b * kCompactWarps, (b + 1) * kCompactWarps), one warp each.
// Its first stream's offset is the sum of every earlier stream's length
// (read by the whole block from L2: at most kFusedMaxStreams lengths), the
// block's own offsets follow from a warp scan, and each warp copies its
// stream.  The last block writes the total and checks the capacity.
constexpr int kCompactWarps = 8;
constexpr int64_t kFusedMaxStreams = 65536;

template <typename Word>
__global__ void __launch_bounds__(kCompactWarps * 32)
    compact_streams_kernel(Geom g, const char *scratch, const uint64_t *lens, uint64_t *offsets,
                           uint8_t *out, uint64_t capacity, int32_t *status) {
  __shared__ unsigned long long part[kCompactWarps];
  __shared__ unsigned long long own[kCompactWarps];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int64_t s0 = (int64_t)blockIdx.x * kCompactWarps;
  // the lengths of streams [0, s0), four loads in flight per thread
  unsigned long long before = 0;
  int64_t i = threadIdx.x;
  for (; i + 3 * (int64_t)blockDim.x < s0; i += 4 * (int64_t)blockDim.x)
    before += __ldg(lens + i) + __ldg(lens + i + blockDim.x) + __ldg(lens + i + 2 * blockDim.x) +
              __ldg(lens + i + 3 * blockDim.x);
  for (; i < s0; i += blockDim.x) before += __ldg(lens + i);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) before += __shfl_xor_sync(kFull, before, o);
  if (lane == 0) part[wid] = before;
  // this block's streams: lane 0 of warp w holds stream s0 + w's length
  const int64_t s = s0 + wid;
  const unsigned long long len = s < g.S ? lens[s] : 0ull;
  if (lane == 0) own[wid] = len;
  __syncthreads();
  unsigned long long base = 0, ex = 0, tot = 0;
  for (int w = 0; w < kCompactWarps; ++w) {
    base += part[w];
    ex += w < wid ? own[w] : 0ull;
    tot += own[w];
  }
  const uint64_t off = base + ex;
  if (s < g.S && lane == 0) offsets[s + 1] = off + len;
  if (blockIdx.x == 0 && threadIdx.x == 0) offsets[0] = 0;
  if (blockIdx.x == gridDim.x - 1 && threadIdx.x == 0 && base + tot > capacity)
    report(status, RANS_ERR_CAPACITY, -1);
  if (s >= g.S) return;
  const StreamDesc d = stream_desc(g, s);
  if (!d.ok || off + len > capacity) return;
  const Word *src = reinterpret_cast<const Word *>(scratch + slot_end(g, d, s) - len);
  Word *dst = reinterpret_cast<Word *>(out + off);
  const uint64_t words = len / sizeof(Word);
  warp_copy_words(dst, src, words);
}

__global__ void debug_divide_kernel(const uint64_t *x, const uint32_t *f, int64_t n, uint64_t *q,
                                    uint32_t *r) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    uint64_t qq;
    uint32_t rr;
    divmod_freq(x[i], f[i], freq_reciprocal(f[i]), qq, rr);
    q[i] = qq;
    r[i] = rr;
  }
}

template <class F, int W, typename SymT, int MODE, bool IB0, bool FLT>
int launch_encode_t(const EncCtx &c, cudaStream_t st) {
  auto kern = encode_kernel<F, W, SymT, MODE, IB0, FLT>;
  const uint32_t tab = enc_table_bytes(MODE, c);
  const uint32_t per_warp = W == 32 ? enc_stage_bytes_per_warp(FLT) : 0;
  uint32_t smem = tab;
  int dev = 0;
  cudaGetDevice(&dev);
  // float latents: the scale table goes after the stage rings when it fits
  const uint32_t tbl = FLT ? (uint32_t)pad16(4ull * (uint64_t)c.K) : 0u;
  const int optin = smem_optin(dev);
  const uint32_t lim = (uint32_t)optin - 64u;  // room for the kernel's static shared memory
  const uint32_t max_dyn = tab + kEncStageBytes + tbl <= lim ? tab + kEncStageBytes + tbl : lim;
  if (ensure_dyn_smem((const void *)kern, (uint32_t)(max_dyn)) !=
      cudaSuccess)
    return RANS_ERR_CUDA;
  const int sms = num_sms(dev);
  int threads;
  int64_t blocks;
  if (W == 32) {
    // Spread the streams over every SM: as many CTAs as fit per SM, each with
    // enough warps for one stream per warp when possible.
    int per_sm = 0;
    if (blocks_per_sm(&per_sm, (const void *)kern, 32, (uint32_t)(tab + per_warp)) !=
            cudaSuccess ||
        per_sm < 1)
      return RANS_ERR_CUDA;
    int64_t nblk = (int64_t)sms * per_sm;
    if (nblk > c.g.S) nblk = c.g.S < 1 ? 1 : c.g.S;
    int64_t warps = (c.g.S + nblk - 1) / nblk;
    if (warps > kEncMaxWarps) warps = kEncMaxWarps;
    // large staged tables leave room for fewer rings
    const int64_t room = ((int64_t)lim - (int64_t)tab) / (int64_t)(per_warp ? per_warp : 1u);
    if (warps > room) warps = room;
    if (warps < 1) return RANS_ERR_CAPACITY;
    threads = (int)warps * 32;
    smem = tab + (uint32_t)warps * per_warp;
    int fit = 0;
    if (blocks_per_sm(&fit, (const void *)kern, threads, (uint32_t)(smem)) != cudaSuccess ||
        fit < 1)
      return RANS_ERR_CUDA;
    const int64_t need = (c.g.S + warps - 1) / warps;
    const int64_t cap = (int64_t)fit * sms;
    blocks = need < cap ? need : cap;
  } else {
    threads = kEncThreads1;
    int fit = 0;
    if (blocks_per_sm(&fit, (const void *)kern, threads, (uint32_t)(smem)) != cudaSuccess ||
        fit < 1)
      return RANS_ERR_CUDA;
    const int64_t need = (c.g.S + threads - 1) / threads;
    const int64_t cap = (int64_t)fit * sms;
    blocks = need < cap ? need : cap;
  }
  if (blocks < 1) blocks = 1;
  EncCtx cc = c;
  cc.stab_smem = tbl > 0 && smem + tbl <= max_dyn ? 1 : 0;
  if (cc.stab_smem) smem += tbl;
  kern<<<(unsigned)blocks, threads, smem, st>>>(cc);
  return cudaGetLastError() == cudaSuccess ? RANS_OK : RANS_ERR_CUDA;
}

template <class F, typename SymT, bool ALIAS>
int launch_encode_wn(const EncCtx &c, int mode, cudaStream_t st) {
  auto kern = encode_kernel_wn<F, SymT, ALIAS>;
  const uint32_t tab = enc_table_bytes(mode, c);
  int dev = 0;
  cudaGetDevice(&dev);
  if (ensure_dyn_smem((const void *)kern, (uint32_t)(tab)) !=
      cudaSuccess)
    return RANS_ERR_CUDA;
  int fit = 0;
  if (blocks_per_sm(&fit, (const void *)kern, kSegThreads, (uint32_t)(tab)) !=
          cudaSuccess ||
      fit < 1)
    return RANS_ERR_CUDA;
  const int64_t warps = (c.g.S + 32 / c.g.W - 1) / (32 / c.g.W);
  const int64_t need = (warps + kSegThreads / 32 - 1) / (kSegThreads / 32);
  const int64_t cap = (int64_t)fit * num_sms(dev);
  int64_t blocks = need < cap ? need : cap;
  if (blocks < 1) blocks = 1;
  kern<<<(unsigned)blocks, kSegThreads, tab, st>>>(c, mode);
  return cudaGetLastError() == cudaSuccess ? RANS_OK : RANS_ERR_CUDA;
}

template <class F, int W, typename SymT, int MODE>
int launch_encode_m(const EncCtx &c, cudaStream_t st) {
  return c.g.ib_shift == 0 ? launch_encode_t<F, W, SymT, MODE, true, false>(c, st)
                           : launch_encode_t<F, W, SymT, MODE, false, false>(c, st);
}

template <class F, int W, typename SymT>
int launch_encode_w(const EncCtx &c, int mode, cudaStream_t st) {
  if (mode == 1) return launch_encode_m<F, W, SymT, 1>(c, st);
  if (mode == 2) return launch_encode_m<F, W, SymT, 2>(c, st);
  return launch_encode_m<F, W, SymT, 0>(c, st);
}

template <class F, typename SymT>
int launch_encode_f(const EncCtx &c, int mode, cudaStream_t st) {
  if (c.g.alias) return launch_encode_wn<F, SymT, true>(c, mode, st);  // W = 1, 2, 4, 8
  if (c.g.W == 32) return launch_encode_w<F, 32, SymT>(c, mode, st);
  if (c.g.W == 1) return launch_encode_w<F, 1, SymT>(c, mode, st);
  return launch_encode_wn<F, SymT, false>(c, mode, st);
}

template <typename SymT>
int launch_encode_s(const EncCtx &c, int mode, cudaStream_t st) {
  return c.g.fmt == RANS_FMT_RANS32_16 ? launch_encode_f<Rans32, SymT>(c, mode, st)
                                       : launch_encode_f<Rans64, SymT>(c, mode, st);
}

}  // namespace

int launch_encode(const void *symbols, int sym_dtype, const int32_t *indexes,
                  const rans_tables &t, const Geom &g, char *scratch, uint64_t *lens,
                  int32_t *status, cudaStream_t st) {
  EncCtx c;
  c.sym = symbols;
  c.idx = indexes;
  c.K = t.K;
  c.sh = (uint32_t)(kPrec - t.precision);
  c.remap = g.alias ? reinterpret_cast<const uint16_t *>(
                          reinterpret_cast<const char *>(t.alias) + t.alias_remap_offset)
                    : nullptr;
  c.meta_bytes = t.meta_bytes;
  c.bucket_bytes = t.bucket_bytes;
  c.start_bytes = t.start_bytes;
  c.blob = reinterpret_cast<const char *>(t.blob);
  c.g = g;
  c.scratch = scratch;
  c.lens = lens;
  c.status = status;
  c.fy = c.fmean = c.fscale = c.stab = nullptr;
  c.bound = 0.0f;
  c.stab_smem = 0;
  const int mode = t.enc_in_smem;
  if (enc_chunk_path_ok(c, mode, sym_dtype, symbols)) {
    const bool per = g.ib_shift == 0;
    const int r = sym_dtype == RANS_SYM_UINT8
                      ? (per ? launch_encode_chunk<uint8_t, true>(c, mode, st)
                             : launch_encode_chunk<uint8_t, false>(c, mode, st))
                  : sym_dtype == RANS_SYM_INT16
                      ? (per ? launch_encode_chunk<int16_t, true>(c, mode, st)
                             : launch_encode_chunk<int16_t, false>(c, mode, st))
                      : (per ? launch_encode_chunk<int32_t, true>(c, mode, st)
                             : launch_encode_chunk<int32_t, false>(c, mode, st));
    if (r != kNotTaken) return r;
  }
  if (enc_tile_path_ok(c, mode, sym_dtype, indexes, symbols)) {
    const int r = g.fmt == RANS_FMT_RANS32_16
                      ? launch_encode_tile<Rans32>(c, mode, indexes, symbols, st)
                      : launch_encode_tile<Rans64>(c, mode, indexes, symbols, st);
    if (r != kNotTaken) return r;
  }
  switch (sym_dtype) {
    case RANS_SYM_INT32: return launch_encode_s<int32_t>(c, mode, st);
    case RANS_SYM_UINT8: return launch_encode_s<uint8_t>(c, mode, st);
    case RANS_SYM_INT16: return launch_encode_s<int16_t>(c, mode, st);
    default: return RANS_ERR_ARG;
  }
}

int launch_encode_float(const float *y, const float *means, const float *scales,
                        const float *scale_table, float scale_bound, const rans_tables &t,
                        const Geom &g, char *scratch, uint64_t *lens, int32_t *status,
                        cudaStream_t st) {
  EncCtx c;
  c.sym = nullptr;
  c.idx = nullptr;
  c.fy = y;
  c.fmean = means;
  c.fscale = scales;
  c.stab = scale_table;
  c.bound = scale_bound;
  c.K = t.K;
  c.sh = 0;
  c.remap = nullptr;
  c.meta_bytes = t.meta_bytes;
  c.bucket_bytes = t.bucket_bytes;
  c.start_bytes = t.start_bytes;
  c.blob = reinterpret_cast<const char *>(t.blob);
  c.g = g;
  c.scratch = scratch;
  c.lens = lens;
  c.status = status;
  // float latents code the 64-bit format only (the caller checks); tiled
  // streams of 64- and 56-wide tiles take the tile-staged kernel (scales and
  // y staged as the index and symbol tiles)
  if ((t.enc_in_smem == 1 || t.enc_in_smem == 2) && flt_tile_shape_ok(g, y, scales)) {
    const int r = launch_encode_tile<Rans64, true>(c, t.enc_in_smem, reinterpret_cast<const int32_t *>(scales), y, st);
    if (r != kNotTaken) return r;
  }
  // tables too large for the bucket words in shared memory are read from
  // global memory here
  const bool smem = t.enc_in_smem == 1;
  if (g.W == 32)
    return smem ? launch_encode_t<Rans64, 32, int32_t, 1, true, true>(c, st)
                : launch_encode_t<Rans64, 32, int32_t, 0, true, true>(c, st);
  return smem ? launch_encode_t<Rans64, 1, int32_t, 1, true, true>(c, st)
              : launch_encode_t<Rans64, 1, int32_t, 0, true, true>(c, st);
}

int launch_compact(const Geom &g, const char *scratch, const uint64_t *lens, uint8_t *out,
                   uint64_t out_capacity, uint64_t *offsets, int32_t *status,
                   cudaStream_t st) {
  if (g.S > 0 && g.S <= kFusedMaxStreams) {
    const unsigned blocks = (unsigned)((g.S + kCompactWarps - 1) / kCompactWarps);
    if (g.fmt == RANS_FMT_RANS32_16)
      compact_streams_kernel<uint16_t><<<blocks, kCompactWarps * 32, 0, st>>>(
          g, scratch, lens, offsets, out, out_capacity, status);
    else
      compact_streams_kernel<uint32_t><<<blocks, kCompactWarps * 32, 0, st>>>(
          g, scratch, lens, offsets, out, out_capacity, status);
    return cudaGetLastError() == cudaSuccess ? RANS_OK : RANS_ERR_CUDA;
  }
  scan_lengths_kernel<<<1, kScanThreads, 0, st>>>(lens, g.S, offsets, out_capacity, status);
  if (g.S > 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    int64_t blocks = (g.S + 7) / 8;
    const int64_t cap = 8LL * num_sms(dev);
    if (blocks > cap) blocks = cap;
    if (g.fmt == RANS_FMT_RANS32_16)
      copy_streams_kernel<uint16_t><<<(unsigned)blocks, 256, 0, st>>>(g, scratch, lens, offsets,
                                                                      out, out_capacity);
    else
      copy_streams_kernel<uint32_t><<<(unsigned)blocks, 256, 0, st>>>(g, scratch, lens, offsets,
                                                                      out, out_capacity);
  }
  return cudaGetLastError() == cudaSuccess ? RANS_OK : RANS_ERR_CUDA;
}

int launch_debug_divide(const uint64_t *x, const uint32_t *f, int64_t n, uint64_t *q,
                        uint32_t *r, cudaStream_t st) {
  if (n <= 0) return RANS_OK;
  int64_t blocks = (n + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  debug_divide_kernel<<<(unsigned)blocks, 256, 0, st>>>(x, f, n, q, r);
  return cudaGetLastError() == cudaSuccess ? RANS_OK : RANS_ERR_CUDA;
}

}  // namespace rb
