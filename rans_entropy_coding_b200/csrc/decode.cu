// decode.cu -- decode_with_indexes.
//
//  * symbol lookup: the decoded bucket is the row's last bucket whose CDF
//    entry is <= cum = x mod 2^16 (the rule of CompressAI's linear scan,
//    "Benchmark notes" section 4).  It is found through a per-row table of
//    2^q slots keyed by the top q bits of cum ("torch_ans 0.3.0", Usage,
//    inverse-CDF decoding): a slot resolves up to two bucket boundaries with
//    two compares, and a slot with more points to boundary bitmaps that a
//    population count resolves; only a table that ran out of bitmap room
//    searches;
//  * state update x = freq (x >> 16) + cum - start and a refill of one
//    32-bit word when x < 2^31 (64-bit state / 32-bit words / 16-bit
//    precision: "torch_ans 0.3.0", Usage, rans64 row); for the rans32_16
//    format (same table, rans32_16 row) cum = x mod 2^p,
//    x = freq (x >> p) + cum - start and a refill of one 16-bit word when
//    x < 2^16 (the F template parameter: Rans64 / Rans32 in rans_common.cuh;
//    the tables hold 16-bit-scaled entries, so the lookup takes cum << sh);
//  * W = 32: one warp per stream, lane = symbol index mod 32; refills take
//    the next words of the shared stream in lane order (ballot + popc)
//    ("torch_ans 0.3.0", Usage legend: warp renormalisation with one shared
//    cursor), served from a 512-word ring in shared memory refilled by
//    cp.async (the 64-bit format's tile and chunk decoders) or from a
//    register buffer of 64 prefetched words (the others);
//  * escapes run off the fast path: lanes proceed one by one in ascending
//    order, reading their bypass pieces, since how many words a lane takes
//    depends on what it reads ("torch_ans 0.3.0", Performance Tuning, GPU
//    item 5: the bypass phase is sequential across the lanes and skipped by a
//    group ballot).  The group is first decoded as if nothing escaped; the
//    ballot, taken beside the refill, sends it down the slow path.
//  Staging: tiled streams move their row indexes in and their values out as
//  tensor-tile copies (decode_tile_kernel), contiguous streams of whole
//  256-symbol chunks with a row per chunk their values out as bulk copies
//  (decode_chunk_kernel); the general kernel streams row indexes through a
//  per-warp shared-memory ring filled with cp.async kDecStage - 1 groups
//  ahead.  Each stream's words are bulk prefetched into L2 when the warp
//  starts it, and tables are staged into shared memory with bulk copies
//  when they fit.
#include <type_traits>

#include <cuda.h>  // CUtensorMap

#include "rans_common.cuh"
#include "rans_internal.h"

namespace rb {
namespace {

constexpr int kDecMaxThreads32 = kDecMaxWarps * 32;
constexpr int kDecThreads1 = 128;

struct DecCtx {
  const uint8_t *in;
  uint64_t in_bytes;
  const uint64_t *offs;
  const int32_t *idx;
  int32_t K;
  uint32_t sh;  // 16 - precision of the rows (Rans32; 0 for Rans64)
  const uint2 *aslots;  // alias coding: the slot words (at the bucket indexes)
  uint32_t meta_bytes, bucket_bytes, start_bytes, slot_bytes;
  const char *blob;
  Geom g;
  void *out;
  int32_t *status;
  // float latents: rows from scales (one per element) and values
  // float(symbol) + mean written to `out` as float
  const float *fscale, *fmean, *stab;
  float bound;
  int32_t stab_smem;  // 1: the kernel copies the scale table into shared memory
};

// A stream's words: its byte range must be word-aligned and hold at least
// the W flushed states (two words each).
template <class F>
__device__ __forceinline__ bool stream_bounds(const DecCtx &c, int64_t s, int W,
                                              const typename F::Word *&words, uint64_t &nw) {
  constexpr uint64_t kWB = sizeof(typename F::Word);
  const uint64_t b0 = c.offs[s], b1 = c.offs[s + 1];
  if (b1 < b0 || b1 > c.in_bytes || ((b0 | b1) & (kWB - 1)) != 0 || (b1 - b0) < 2 * kWB * W)
    return false;
  words = reinterpret_cast<const typename F::Word *>(c.in + b0);
  nw = (b1 - b0) / kWB;
  return true;
}

// The bucket holding cum in row m: the slot's own two boundaries, or its
// boundary bitmap (the bitmap word is read for every lane, from the slot
// itself when the slot needs none, so the lookup takes no branch).  With
// SEARCH (a table with slots that ran out of bitmap room) those slots take a
// binary search over the starts; WARP: the search is entered once per warp.
template <bool SEARCH, bool WARP>
__device__ __forceinline__ uint32_t lookup(uint32_t cum, const RowMeta &m, const uint16_t *starts,
                                           const uint32_t *slots, bool active) {
  const uint32_t sh = slot_shift(m.slot);
  const uint32_t i1 = slot_base(m.slot) + (cum >> sh);
  const uint32_t se = slots[i1];
  const uint32_t e1 = (se >> 16) & 0xffu, e2 = se >> 24;
  const uint32_t c = cum & ((1u << sh) - 1u);
  const uint32_t lo = se & 0xffffu;
  uint32_t sym = lo + (c > e1 ? 1u : 0u) + (c > e2 ? 1u : 0u);
  const bool bitmap = e1 == 0xffu && e2 != 0xffu;
  const uint32_t i2 = bitmap ? (lo | ((se >> 8) & 0xff0000u)) + (c >> 4) : i1;
  const uint32_t ce = slots[i2];
  const uint32_t sym2 = (ce >> 16) + __popc(ce & ((2u << (c & 15u)) - 1u));
  sym = bitmap ? sym2 : sym;
  if (SEARCH) {
    const bool srch = active && e1 > e2 && e1 != 0xffu;
    if (WARP ? __any_sync(kFull, srch) : srch) {
      if (srch) {  // last bucket in [lo, lo + e2 + 3] whose start is <= cum
        uint32_t l = lo, h = lo + e2 + 3u;
        while (l < h) {
          const uint32_t mid = (l + h + 1) >> 1;
          if (starts[m.bucket_base + mid] <= cum) l = mid; else h = mid - 1;
        }
        sym = l;
      }
    }
  }
  // never past the row's last bucket, whatever the slots hold (a refresh that
  // rejected a row leaves that row's slots stale)
  return min(sym, m.maxv);
}

// The bucket holding cum when the row's slots are not on chip: the last of
// the row's maxv + 1 buckets whose start is <= cum, by a binary search over
// its 16-bit starts in power-of-two steps (every probe is in the row; the
// row end is never read).
__device__ __forceinline__ uint32_t search_row(uint32_t cum, const RowMeta &m,
                                               const uint16_t *starts) {
  const uint32_t last = m.maxv;  // buckets 0 .. maxv
  const uint16_t *row = starts + m.bucket_base;
  uint32_t j = 0;
  for (uint32_t step = last ? 1u << (31 - __clz(last)) : 0u; step != 0; step >>= 1) {
    const uint32_t t = j + step;
    const uint32_t v = row[t <= last ? t : last];
    j = (t <= last && v <= cum) ? t : j;
  }
  return j;
}

template <class F>
struct EscapeResult {
  typename F::State x;
  int64_t val;
  uint64_t cur;
  bool bad;
};

// The lane-serial part of a group holding an escape (after every lane's
// symbol op): lanes take their words in ascending lane order; an escaping lane
// reads its refill, count pieces and bypass pieces from the shared stream.
template <class F>
__device__ __forceinline__ EscapeResult<F> escape_group(typename F::State x, bool active,
                                                     bool esc, uint32_t maxv, uint64_t abs0,
                                                     const typename F::Word *words,
                                                     uint64_t nw) {
  const int lane = threadIdx.x & 31;
  bool bad = false;
  int64_t val = 0;
  const bool need_sym = active && x < F::kLow;
  uint32_t cons = need_sym ? 1u : 0u;
  uint32_t rem = __ballot_sync(kFull, esc);
  while (rem) {
    const int el = __ffs(rem) - 1;
    rem &= rem - 1;
    uint32_t inc = cons;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(kFull, inc, o);
      if (lane >= o) inc += t;
    }
    const uint32_t pre = __shfl_sync(kFull, inc - cons, el);
    if (lane == el) {
      uint64_t pp = abs0 + pre;
      auto rd = [&]() -> uint32_t {
        uint32_t v = 0;
        if (pp < nw) v = __ldg(words + pp); else bad = true;
        ++pp;
        return v;
      };
      if (x < F::kLow) x = (x << F::kWordBits) | rd();
      auto getbits = [&]() -> uint32_t {
        const uint32_t v = (uint32_t)x & kBypassMax;
        x >>= kBypassBits;
        if (x < F::kLow) x = (x << F::kWordBits) | rd();
        return v;
      };
      uint32_t v4 = getbits();
      uint32_t nb = v4;
      while (v4 == kBypassMax && nb <= 15) {
        v4 = getbits();
        nb += v4;
      }
      if (nb > 15) {
        bad = true;
        nb = 0;
      }
      uint64_t raw = 0;
      for (uint32_t k = 0; k < nb; ++k) raw |= (uint64_t)getbits() << (kBypassBits * k);
      const int64_t half = (int64_t)(raw >> 1);
      val = (raw & 1) ? (-half - 1) : ((int64_t)maxv + half);
      cons = (uint32_t)(pp - (abs0 + pre));
    }
  }
  uint32_t inc = cons;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(kFull, inc, o);
    if (lane >= o) inc += t;
  }
  if (need_sym && !esc) {
    const uint64_t pp = abs0 + (inc - cons);
    uint32_t v = 0;
    if (pp < nw) v = __ldg(words + pp); else bad = true;
    x = (x << F::kWordBits) | v;
  }
  EscapeResult<F> r;
  r.x = x;
  r.val = val;
  r.cur = abs0 + __shfl_sync(kFull, inc, 31);
  r.bad = bad;
  return r;
}

// Per-warp decoder state for one stream.
template <class F>
struct WarpDec {
  typename F::State x;   // this lane's state
  uint64_t cur;          // absolute word index of the register window
  uint32_t off;          // words of the window already consumed (< 32)
  uint32_t w0, w1, w2;   // window words cur + lane, + 32, + 64 (w2: lookahead)
  uint32_t rmax;         // largest row index seen (checked once per stream)
  bool bad;
};

// Window word i, read from a clamped address (nw >= 64 always): reading past
// the stream end returns its last word instead, so no select waits on the
// load; a decoder that consumes past the end is caught by the final check.
template <typename Word>
__device__ __forceinline__ uint32_t word_at(const Word *words, uint64_t nw, uint64_t i) {
  return __ldg(words + (i < nw ? i : nw - 1));
}

template <class F>
__device__ __forceinline__ void load_window(WarpDec<F> &st, const typename F::Word *words,
                                            uint64_t nw) {
  const int lane = threadIdx.x & 31;
  st.w0 = word_at(words, nw, st.cur + lane);
  st.w1 = word_at(words, nw, st.cur + 32 + lane);
  st.w2 = word_at(words, nw, st.cur + 64 + lane);
}

// One group of 32 symbols: lookup, state update, refill, output.  m is the
// group's row metadata, read one group ahead.  The refill is taken as if no
// lane escaped; the escape ballot, issued beside it, sends the group down
// the lane-serial path from the state after the symbol op.
template <class F, typename SymT, bool FULL, bool SEARCH, bool ROWS>
__device__ __forceinline__ void dec_group(WarpDec<F> &st, const RowMeta &m,
                                          const uint16_t *starts, const uint32_t *slots,
                                          bool active, SymT *dst, const typename F::Word *words,
                                          uint64_t nw, uint32_t sh, float mean = 0.0f) {
  const int lane = threadIdx.x & 31;
  if (FULL) active = true;
  const uint32_t cum = F::cum16(st.x, sh);
  const uint32_t sym =
      ROWS ? search_row(cum, m, starts) : lookup<SEARCH, true>(cum, m, starts, slots, active);
  const uint32_t start = starts[m.bucket_base + sym];
  const uint32_t freq = width_of(start, starts[m.bucket_base + sym + 1]);
  typename F::State x = F::dec_step(st.x, cum, start, freq, sh);
  if (!FULL) x = active ? x : st.x;
  const bool esc = active && sym == m.maxv;
  const bool need = active && x < F::kLow;
  const uint32_t nm = __ballot_sync(kFull, need);
  const bool any_esc = __any_sync(kFull, esc);
  const uint32_t j = st.off + __popc(nm & lanemask_lt());
  // the lane holding window word j (mod 32) sends it from w0 or w1
  const uint32_t wv = __shfl_sync(kFull, (uint32_t)lane >= st.off ? st.w0 : st.w1, j & 31);
  int32_t val = (int32_t)sym + m.offset;
  if (!any_esc) {
    st.x = need ? ((x << F::kWordBits) | wv) : x;
    st.off += __popc(nm);
    if (st.off >= 32) {
      st.w0 = st.w1;
      st.w1 = st.w2;
      st.cur += 32;
      st.off -= 32;
      st.w2 = word_at(words, nw, st.cur + 64 + lane);
    }
  } else {
    const EscapeResult<F> er =
        escape_group<F>(x, active, esc, m.maxv, st.cur + st.off, words, nw);
    st.x = er.x;
    if (esc) val = (int32_t)(er.val + (int64_t)m.offset);
    st.bad |= er.bad;
    st.cur = er.cur;
    st.off = 0;
    load_window(st, words, nw);
  }
  if (active) {
    if (std::is_same<SymT, float>::value) st_global(dst, (SymT)((float)val + mean));
    else st_global(dst, (SymT)val);
  }
}

// One warp decodes one stream, a group of 32 symbols per step: the copies
// for group g + kDecStage - 1, group g+1's row metadata from the ring, then
// group g's decode.
// SymT = float: the ring holds scales, each group's row is its scale's table
// row, and the output is float(symbol) + mean, the means read one group
// ahead with plain loads.
template <class F, typename SymT, bool IB0, bool WIDE, bool SEARCH, bool ROWS>
__device__ __forceinline__ void decode_stream_w32(const DecCtx &c, const StreamDesc &d,
                                                  const RowMeta *meta, const uint16_t *starts,
                                                  const uint32_t *slots, uint32_t *stg,
                                                  int64_t s, const typename F::Word *words,
                                                  uint64_t nw, const float *stab) {
  using State = typename F::State;
  constexpr int kS = kDecStage;
  const int lane = threadIdx.x & 31;
  const int32_t n = (int32_t)d.n;
  const int32_t G = (n + 31) >> 5;
  const int64_t base = d.base;
  const int ib = c.g.ib_shift;
  const int32_t *idx_s = c.idx + (IB0 ? base : 0);
  SymT *out_s = reinterpret_cast<SymT *>(c.out) + base;
  const uint32_t kmax = (uint32_t)c.K - 1u;
  const uint32_t sh = F::shift(c.sh);

  WarpDec<F> st;
  st.x = (State)__ldg(words + 2 * lane) | ((State)__ldg(words + 2 * lane + 1) << F::kWordBits);
  st.cur = 64;
  st.off = 0;
  load_window(st, words, nw);
  st.rmax = 0;
  st.bad = false;

  // Group g's row indexes land in stage slot g mod kS, copied kS - 1 groups
  // ahead.  Copies for groups past the end (and lanes past the stream end)
  // read the stream's element 0 and are never used.
  Stepper<WIDE> pl;  // next group to copy
  pl.init(d.t, lane);
  Stepper<WIDE> pc = pl;  // group being decoded (output position)
  constexpr bool kFlt = std::is_same<SymT, float>::value;
  const float *fs_s = kFlt ? c.fscale + base : nullptr;
  const float *fm_s = kFlt && c.fmean ? c.fmean + base : nullptr;
  auto issue = [&](int32_t gi) {
    const int32_t rel = gi < G && lane < n - gi * 32 ? pl.rel : 0;
    if (kFlt) {
      cp_async4(stg + (gi & (kS - 1)) * 32 + lane, fs_s + rel);
      if (fm_s) prefetch_l2(fm_s + rel);
    } else {
      cp_async4(stg + (gi & (kS - 1)) * 32 + lane,
                IB0 ? idx_s + rel : c.idx + ((base + rel) >> ib));
    }
    cp_async_commit();
    pl.fwd(32);
  };
  auto meta_of = [&](uint32_t v) -> RowMeta {
    const uint32_t r =
        kFlt ? scale_row(bound_scale(__uint_as_float(v), c.bound), stab, c.K) : v;
    st.rmax = max(st.rmax, r);
    return row_meta(meta, min(r, kmax));
  };
  // the mean of group g's element for this lane (0 past the stream end)
  auto mean_at = [&](int32_t g, int32_t rel) -> float {
    return fm_s && g < G && lane < n - g * 32 ? __ldg(fm_s + rel) : 0.0f;
  };
#pragma unroll 1
  for (int32_t u = 0; u < kS - 1; ++u) issue(u);
  cp_async_wait<kS - 2>();
  RowMeta m = meta_of(stg[lane]);
  // float values: means read two groups ahead (pm: position of the next)
  Stepper<WIDE> pm = pc;
  float mean = kFlt ? mean_at(0, pm.rel) : 0.0f;
  if (kFlt) pm.fwd(32);
  float mean_n = kFlt ? mean_at(1, pm.rel) : 0.0f;
  if (kFlt) pm.fwd(32);
#pragma unroll 1
  for (int32_t g = 0; g + 1 < G; ++g) {
    issue(g + kS - 1);
    cp_async_wait<kS - 2>();  // groups up to g + 1 have landed
    const RowMeta mn = meta_of(stg[((g + 1) & (kS - 1)) * 32 + lane]);
    const float mean_nn = kFlt ? mean_at(g + 2, pm.rel) : 0.0f;
    if (kFlt) pm.fwd(32);
    dec_group<F, SymT, true, SEARCH, ROWS>(st, m, starts, slots, true, out_s + pc.rel, words,
                                           nw, sh, mean);
    pc.fwd(32);
    m = mn;
    mean = mean_n;
    mean_n = mean_nn;
  }
  dec_group<F, SymT, false, SEARCH, ROWS>(st, m, starts, slots, lane < n - (G - 1) * 32,
                                          out_s + pc.rel, words, nw, sh, mean);
  cp_async_wait<0>();
  if (__any_sync(kFull, st.rmax > kmax)) {
    if (lane == 0) report(c.status, RANS_ERR_INDEX, s);
    return;
  }
  const bool ok = !st.bad && st.x == F::kLow && st.cur + st.off == nw;
  if (!__all_sync(kFull, ok) && lane == 0) report(c.status, RANS_ERR_CORRUPT, s);
}

template <class F, typename SymT, bool IB0, bool SEARCH, bool ROWS>
__device__ __forceinline__ void decode_stream_w32_entry(const DecCtx &c, const RowMeta *meta,
                                                        const uint16_t *buckets,
                                                        const uint32_t *slots, uint32_t *stg,
                                                        int64_t s, const float *stab) {
  using State = typename F::State;
  using Word = typename F::Word;
  const int lane = threadIdx.x & 31;
  const StreamDesc d = stream_desc(c.g, s);
  const Word *words = nullptr;
  uint64_t nw = 0;
  if (!d.ok || !stream_bounds<F>(c, s, 32, words, nw)) {
    if (lane == 0) report(c.status, d.ok ? RANS_ERR_CORRUPT : RANS_ERR_ARG, s);
    return;
  }
  if (lane == 0)
    bulk_prefetch_l2(reinterpret_cast<const char *>(c.in),
                     reinterpret_cast<const char *>(c.in) + c.in_bytes,
                     reinterpret_cast<const char *>(words + 64), sizeof(Word) * (nw - 64));
  if (d.n == 0) {  // only the 32 initial states
    const State x =
        (State)__ldg(words + 2 * lane) | ((State)__ldg(words + 2 * lane + 1) << F::kWordBits);
    if (!__all_sync(kFull, x == F::kLow && nw == 64) && lane == 0)
      report(c.status, RANS_ERR_CORRUPT, s);
    return;
  }
  if (d.t.ww >= 32)
    decode_stream_w32<F, SymT, IB0, true, SEARCH, ROWS>(c, d, meta, buckets, slots, stg, s,
                                                        words, nw, stab);
  else
    decode_stream_w32<F, SymT, IB0, false, SEARCH, ROWS>(c, d, meta, buckets, slots, stg, s,
                                                         words, nw, stab);
}

template <class F, typename SymT, bool ROWS>
__device__ void decode_stream_w1(const DecCtx &c, const RowMeta *meta, const uint16_t *buckets,
                                 const uint32_t *slots, int64_t s, const float *stab) {
  using State = typename F::State;
  using Word = typename F::Word;
  const StreamDesc d = stream_desc(c.g, s);
  const Word *words = nullptr;
  uint64_t nw = 0;
  if (!d.ok || !stream_bounds<F>(c, s, 1, words, nw)) {
    report(c.status, d.ok ? RANS_ERR_CORRUPT : RANS_ERR_ARG, s);
    return;
  }
  bulk_prefetch_l2(reinterpret_cast<const char *>(c.in),
                   reinterpret_cast<const char *>(c.in) + c.in_bytes,
                   reinterpret_cast<const char *>(words), sizeof(Word) * nw);
  const uint32_t sh = F::shift(c.sh);
  const int ib = c.g.ib_shift;
  const Tile t = d.t;
  State x = (State)__ldg(words) | ((State)__ldg(words + 1) << F::kWordBits);
  uint64_t pw = 2;  // words consumed
  bool bad = false;
  // the next four words wait in registers, each loaded four refills before
  // it is used, so that a refill does not wait on memory (loads past the
  // stream's end read its last word; consuming past it is an error)
  uint32_t wq[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) wq[u] = __ldg(words + (2 + u < nw ? 2 + u : nw - 1));
  auto rd = [&]() -> uint32_t {
    const uint32_t v = wq[0];
    bad |= pw >= nw;
    wq[0] = wq[1];
    wq[1] = wq[2];
    wq[2] = wq[3];
    const uint64_t q = pw + 4;
    wq[3] = __ldg(words + (q < nw ? q : nw - 1));
    ++pw;
    return v;
  };
  RelPos pl, pp;
  pl.init(t, 0);
  pp = pl;
  const int32_t n = (int32_t)d.n;
  constexpr int32_t kAhead = 64;
  constexpr bool kFlt = std::is_same<SymT, float>::value;
  auto prefetch = [&](int64_t q) {
    if (kFlt) prefetch_l2(c.fscale + q);
    else prefetch_l2(c.idx + (q >> ib));
  };
  for (int32_t u = 0; u < kAhead && u < n; ++u) {
    prefetch(d.base + pp.rel(t));
    pp.fwd(t, 1);
  }
  // The rows (and, for float values, the means) of the next kRing symbols
  // wait in registers, each read kRing symbols before it is decoded, so
  // that the state chain does not wait on their loads.
  constexpr int kRing = 4;
  RelPos pf = pl;  // next symbol to fetch into the ring
  int32_t rrow[kRing];
  float rmean[kRing];
  auto fetch = [&](int32_t &r, float &mean) {
    const int64_t q = d.base + pf.rel(t);
    pf.fwd(t, 1);
    r = kFlt ? (int32_t)scale_row(bound_scale(__ldg(c.fscale + q), c.bound), stab, c.K)
             : __ldg(c.idx + (q >> ib));
    mean = kFlt && c.fmean ? __ldg(c.fmean + q) : 0.0f;
  };
#pragma unroll
  for (int u = 0; u < kRing; ++u) {
    rrow[u] = 0;
    rmean[u] = 0.0f;
    if (u < n) fetch(rrow[u], rmean[u]);
  }
  // the row metadata of the next symbol, read one symbol ahead (clamped to
  // the table; an out-of-range row is reported when its symbol comes)
  const uint32_t kmax = (uint32_t)c.K - 1u;
  RowMeta m_next = row_meta(meta, min((uint32_t)rrow[0], kmax));
  for (int32_t i = 0; i < n; ++i) {
    const int64_t p = d.base + pl.rel(t);
    pl.fwd(t, 1);
    const int32_t r = rrow[0];
    const float mean_i = rmean[0];
#pragma unroll
    for (int u = 0; u + 1 < kRing; ++u) {
      rrow[u] = rrow[u + 1];
      rmean[u] = rmean[u + 1];
    }
    if (i + kRing < n) fetch(rrow[kRing - 1], rmean[kRing - 1]);
    if (i + kAhead < n) {
      prefetch(d.base + pp.rel(t));
      pp.fwd(t, 1);
    }
    if ((uint32_t)r >= (uint32_t)c.K) {
      report(c.status, RANS_ERR_INDEX, s);
      return;
    }
    const RowMeta m = m_next;
    m_next = row_meta(meta, min((uint32_t)rrow[0], kmax));
    const uint32_t cum = F::cum16(x, sh);
    const uint32_t sym =
        ROWS ? search_row(cum, m, buckets) : lookup<true, false>(cum, m, buckets, slots, true);
    const uint32_t start = buckets[m.bucket_base + sym];
    const uint32_t freq = width_of(start, buckets[m.bucket_base + sym + 1]);
    x = F::dec_step(x, cum, start, freq, sh);
    if (x < F::kLow) x = (x << F::kWordBits) | rd();
    int64_t val = (int64_t)sym;
    if (sym == m.maxv) {
      auto getbits = [&]() -> uint32_t {
        const uint32_t v = (uint32_t)x & kBypassMax;
        x >>= kBypassBits;
        if (x < F::kLow) x = (x << F::kWordBits) | rd();
        return v;
      };
      uint32_t v4 = getbits();
      uint32_t nb = v4;
      while (v4 == kBypassMax && nb <= 15) {
        v4 = getbits();
        nb += v4;
      }
      if (nb > 15) {
        bad = true;
        nb = 0;
      }
      uint64_t raw = 0;
      for (uint32_t k = 0; k < nb; ++k) raw |= (uint64_t)getbits() << (kBypassBits * k);
      const int64_t half = (int64_t)(raw >> 1);
      val = (raw & 1) ? (-half - 1) : ((int64_t)m.maxv + half);
    }
    if constexpr (kFlt)
      st_global(reinterpret_cast<float *>(c.out) + p,
                (float)(int32_t)(val + (int64_t)m.offset) + mean_i);
    else
      SymIO<SymT>::store(c.out, p, val + (int64_t)m.offset);
  }
  if (bad || x != F::kLow || pw != nw) report(c.status, RANS_ERR_CORRUPT, s);
}

// One state on a contiguous stream (symbol i of the stream at base + i):
// four symbols a step, their row indexes read a step ahead and their row
// metadata before the first of them is decoded, the stream's next words in
// registers; the symbol step is decode_stream_w1's.
template <class F, typename SymT, bool ROWS>
__device__ void decode_stream_w1c(const DecCtx &c, const RowMeta *meta, const uint16_t *buckets,
                                  const uint32_t *slots, int64_t s) {
  using State = typename F::State;
  using Word = typename F::Word;
  const StreamDesc d = stream_desc(c.g, s);
  const Word *words = nullptr;
  uint64_t nw = 0;
  if (!d.ok || !stream_bounds<F>(c, s, 1, words, nw)) {
    report(c.status, d.ok ? RANS_ERR_CORRUPT : RANS_ERR_ARG, s);
    return;
  }
  bulk_prefetch_l2(reinterpret_cast<const char *>(c.in),
                   reinterpret_cast<const char *>(c.in) + c.in_bytes,
                   reinterpret_cast<const char *>(words), sizeof(Word) * nw);
  const uint32_t sh = F::shift(c.sh);
  const int ib = c.g.ib_shift;
  const int32_t n = (int32_t)d.n;
  const int32_t *idx = c.idx;
  const int64_t base = d.base;
  const uint32_t kmax = (uint32_t)c.K - 1u;
  State x = (State)__ldg(words) | ((State)__ldg(words + 1) << F::kWordBits);
  uint64_t pw = 2;  // words consumed
  bool bad = false;
  uint32_t wq[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) wq[u] = __ldg(words + (2 + u < nw ? 2 + u : nw - 1));
  auto rd = [&]() -> uint32_t {
    const uint32_t v = wq[0];
    bad |= pw >= nw;
    wq[0] = wq[1];
    wq[1] = wq[2];
    wq[2] = wq[3];
    const uint64_t q = pw + 4;
    wq[3] = __ldg(words + (q < nw ? q : nw - 1));
    ++pw;
    return v;
  };
  auto rows4 = [&](int32_t i, int32_t (&r)[4]) {
#pragma unroll
    for (int u = 0; u < 4; ++u) r[u] = i + u < n ? __ldg(idx + ((base + i + u) >> ib)) : 0;
  };
  for (int32_t q = 0; q < 64 && q < n; q += 16) prefetch_l2(idx + ((base + q) >> ib));
  int32_t ra[4], rn[4];
  rows4(0, ra);
  rows4(4, rn);
#pragma unroll 1
  for (int32_t i = 0; i < n; i += 4) {
    RowMeta m[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) m[u] = row_meta(meta, min((uint32_t)ra[u], kmax));
    if ((i & 15) == 0 && i + 64 < n) prefetch_l2(idx + ((base + i + 64) >> ib));
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (i + u >= n) break;
      if ((uint32_t)ra[u] >= (uint32_t)c.K) {
        report(c.status, RANS_ERR_INDEX, s);
        return;
      }
      const uint32_t cum = F::cum16(x, sh);
      const uint32_t sym = ROWS ? search_row(cum, m[u], buckets)
                                : lookup<true, false>(cum, m[u], buckets, slots, true);
      const uint32_t start = buckets[m[u].bucket_base + sym];
      const uint32_t freq = width_of(start, buckets[m[u].bucket_base + sym + 1]);
      x = F::dec_step(x, cum, start, freq, sh);
      if (x < F::kLow) x = (x << F::kWordBits) | rd();
      int64_t val = (int64_t)sym;
      if (sym == m[u].maxv) {
        auto getbits = [&]() -> uint32_t {
          const uint32_t v = (uint32_t)x & kBypassMax;
          x >>= kBypassBits;
          if (x < F::kLow) x = (x << F::kWordBits) | rd();
          return v;
        };
        uint32_t v4 = getbits();
        uint32_t nb = v4;
        while (v4 == kBypassMax && nb <= 15) {
          v4 = getbits();
          nb += v4;
        }
        if (nb > 15) {
          bad = true;
          nb = 0;
        }
        uint64_t raw = 0;
        for (uint32_t k = 0; k < nb; ++k) raw |= (uint64_t)getbits() << (kBypassBits * k);
        const int64_t half = (int64_t)(raw >> 1);
        val = (raw & 1) ? (-half - 1) : ((int64_t)m[u].maxv + half);
      }
      SymIO<SymT>::store(c.out, base + i + u, val + (int64_t)m[u].offset);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) ra[u] = rn[u];
    rows4(i + 8, rn);
  }
  if (bad || x != F::kLow || pw != nw) report(c.status, RANS_ERR_CORRUPT, s);
}

// W = 2, 4 or 8 interleaved states on W consecutive lanes of a warp, 32 / W
// streams per warp ("torch_ans 0.3.0", Usage legend: num_interleaves 2, 4
// and 8 map to that many consecutive lanes, sub-warp groups).  Lane l of a
// segment holds state l and decodes symbols l, l + W, ...; refills take the
// segment's next words in lane order (ballot + popc within the segment's
// lanes); a group holding an escape goes lane by lane in ascending order,
// every segment's scans restarting at its first lane.  All lanes run the
// same number of groups (the warp's longest stream), idle lanes masked.
template <class F>
__device__ __forceinline__ EscapeResult<F> escape_group_seg(
    typename F::State x, bool active, bool esc, uint32_t maxv, uint64_t abs0,
    const typename F::Word *words, uint64_t nw, int l, int W, int seg_last) {
  const int lane = threadIdx.x & 31;
  bool bad = false;
  int64_t val = 0;
  const bool need_sym = active && x < F::kLow;
  uint32_t cons = need_sym ? 1u : 0u;
  auto seg_scan = [&](uint32_t v) {  // inclusive scan over the segment's lanes
    uint32_t inc = v;
    for (int o = 1; o < W; o <<= 1) {
      const uint32_t t = __shfl_up_sync(kFull, inc, o);
      if (l >= o) inc += t;
    }
    return inc;
  };
  uint32_t rem = __ballot_sync(kFull, esc);
  while (rem) {
    const int el = __ffs(rem) - 1;
    rem &= rem - 1;
    const uint32_t inc = seg_scan(cons);
    const uint32_t pre = __shfl_sync(kFull, inc - cons, el);
    if (lane == el) {
      uint64_t pp = abs0 + pre;
      auto rd = [&]() -> uint32_t {
        uint32_t v = 0;
        if (pp < nw) v = __ldg(words + pp); else bad = true;
        ++pp;
        return v;
      };
      if (x < F::kLow) x = (x << F::kWordBits) | rd();
      auto getbits = [&]() -> uint32_t {
        const uint32_t v = (uint32_t)x & kBypassMax;
        x >>= kBypassBits;
        if (x < F::kLow) x = (x << F::kWordBits) | rd();
        return v;
      };
      uint32_t v4 = getbits();
      uint32_t nb = v4;
      while (v4 == kBypassMax && nb <= 15) {
        v4 = getbits();
        nb += v4;
      }
      if (nb > 15) {
        bad = true;
        nb = 0;
      }
      uint64_t raw = 0;
      for (uint32_t k = 0; k < nb; ++k) raw |= (uint64_t)getbits() << (kBypassBits * k);
      const int64_t half = (int64_t)(raw >> 1);
      val = (raw & 1) ? (-half - 1) : ((int64_t)maxv + half);
      cons = (uint32_t)(pp - (abs0 + pre));
    }
  }
  const uint32_t inc = seg_scan(cons);
  if (need_sym && !esc) {
    const uint64_t pp = abs0 + (inc - cons);
    uint32_t v = 0;
    if (pp < nw) v = __ldg(words + pp); else bad = true;
    x = (x << F::kWordBits) | v;
  }
  EscapeResult<F> r;
  r.x = x;
  r.val = val;
  r.cur = abs0 + __shfl_sync(kFull, inc, seg_last);
  r.bad = bad;
  return r;
}

// One segment's stream (s < 0: an idle segment, still taking part in the
// warp's votes and shuffles).  ALIAS: alias-coded streams (the slot of the
// position gives symbol and rank).
template <class F, typename SymT, bool ROWS, bool ALIAS>
__device__ void decode_segment(const DecCtx &c, const RowMeta *meta, const uint16_t *starts,
                               const uint32_t *slots, int64_t s, int W) {
  using State = typename F::State;
  using Word = typename F::Word;
  const int lane = threadIdx.x & 31;
  const int l = lane & (W - 1);
  const int seg0 = lane - l;
  const uint32_t segmask = (W == 32 ? kFull : ((1u << W) - 1u)) << seg0;
  const uint32_t sh = F::shift(c.sh);
  StreamDesc d;
  d.ok = false;
  d.n = 0;
  d.base = 0;
  d.t = Tile{1, kNoWrap, 0, 0};
  const Word *words = nullptr;
  uint64_t nw = 0;
  bool live = false;
  if (s >= 0) {
    d = stream_desc(c.g, s);
    live = d.ok && stream_bounds<F>(c, s, W, words, nw);
    if (!live && l == 0) report(c.status, d.ok ? RANS_ERR_CORRUPT : RANS_ERR_ARG, s);
    if (live && l == 0)
      bulk_prefetch_l2(reinterpret_cast<const char *>(c.in),
                       reinterpret_cast<const char *>(c.in) + c.in_bytes,
                       reinterpret_cast<const char *>(words), sizeof(Word) * nw);
  }
  State x = F::kLow;
  if (live) x = (State)__ldg(words + 2 * l) | ((State)__ldg(words + 2 * l + 1) << F::kWordBits);
  uint64_t cur = 2 * (uint64_t)W;
  const int32_t n = live ? (int32_t)d.n : 0;
  const int32_t G = (n + W - 1) / W;
  const int32_t Gmax = (int32_t)__reduce_max_sync(kFull, (uint32_t)G);
  const int ib = c.g.ib_shift;
  const uint32_t kmax = (uint32_t)c.K - 1u;
  bool bad = false, bad_index = false;
  // the row index of this lane's element in group k, read one group ahead
  auto pos_of = [&](int32_t k) -> int64_t {
    RelPos rp;
    rp.init(d.t, k * W + l);
    return d.base + rp.rel(d.t);
  };
  int32_t rn = 0;
  if (0 < G && l < n) rn = __ldg(c.idx + (pos_of(0) >> ib));
  for (int32_t k = 0; k < Gmax; ++k) {
    const int32_t i = k * W + l;
    const bool active = i < n;
    const uint32_t r = (uint32_t)rn;
    rn = 0;
    if (i + W < n) rn = __ldg(c.idx + (pos_of(k + 1) >> ib));
    bad_index |= active && r > kmax;
    const RowMeta m = row_meta(meta, active && r <= kmax ? r : 0u);
    const uint32_t cum = F::cum16(x, sh);
    uint32_t sym, rank = 0;
    if constexpr (ALIAS) sym = alias_lookup(cum >> sh, m, c.aslots, kPrec - sh, rank);
    else sym = ROWS ? search_row(cum, m, starts) : lookup<true, true>(cum, m, starts, slots, active);
    const uint32_t start = starts[m.bucket_base + sym];
    const uint32_t freq = width_of(start, starts[m.bucket_base + sym + 1]);
    State y = ALIAS ? F::dec_rank_step(x, freq, rank, sh) : F::dec_step(x, cum, start, freq, sh);
    if (!active) y = x;
    const bool esc = active && sym == m.maxv;
    const bool need = active && y < F::kLow;
    const uint32_t nm = __ballot_sync(kFull, need);
    int64_t val = (int64_t)sym;
    if (!__any_sync(kFull, esc)) {
      if (need) {
        const uint64_t pp = cur + __popc(nm & segmask & lanemask_lt());
        uint32_t v = 0;
        if (pp < nw) v = __ldg(words + pp); else bad = true;
        y = (y << F::kWordBits) | v;
      }
      cur += __popc(nm & segmask);
    } else {
      const EscapeResult<F> er =
          escape_group_seg<F>(y, active, esc, m.maxv, cur, words, nw, l, W, seg0 + W - 1);
      y = er.x;
      if (esc) val = er.val;
      bad |= er.bad;
      cur = er.cur;
    }
    x = y;
    if (active) SymIO<SymT>::store(c.out, pos_of(k), val + (int64_t)m.offset);
  }
  // every lane votes (idle segments too), then each live segment's first
  // lane reports
  const bool ok = !live || (!bad && x == F::kLow && cur == nw);
  const uint32_t fails = __ballot_sync(kFull, !ok) & segmask;
  const uint32_t idx_fails = __ballot_sync(kFull, bad_index) & segmask;
  if (live && l == 0 && idx_fails) report(c.status, RANS_ERR_INDEX, s);
  else if (live && l == 0 && fails) report(c.status, RANS_ERR_CORRUPT, s);
}

// Shared-memory bytes of a table mode: 0 reads the tables from global
// memory, 1 stages the row metadata, starts and lookup slots, 2 (tables whose
// slots do not fit) the row metadata and starts, the lookup then searching
// each row's starts.
__host__ __device__ inline uint32_t dec_table_bytes(int mode, const DecCtx &c) {
  return mode == 1 ? c.meta_bytes + c.start_bytes + c.slot_bytes
                   : (mode == 2 ? c.meta_bytes + c.start_bytes : 0u);
}

// ---------------------------------------------- W = 32, tile-staged I/O ----
// Tiled streams whose tile rows are whole 16-byte units go through a leaner
// warp decoder: the row indexes of 4 tile rows of one channel (a chunk of
// ww / 8 groups) arrive in a per-warp shared-memory ring with one
// tensor-tile copy, each decoded value overwrites its row index in the ring,
// and the chunk leaves with one tensor-tile store.  No thread computes an
// element address; the copy engine walks the tile's rows and channels.
// The ring has two halves of 4 rows x up to 64 int32: while chunk k decodes
// from one half, chunk k + 1 lands in the other.  Its load is issued three
// groups before the end of chunk k, when chunk k - 1's store has long read
// that half, and finds the chunk in L2: every chunk is prefetched into L2
// three chunks ahead.
constexpr uint32_t kTileWaitTries = 1u << 22;  // bounded mbarrier waits (about 4 s)

struct TileMaps {
  CUtensorMap idx[2];  // row indexes: box (tile width, 4, 1); [1]: last tile column
  CUtensorMap out[2];  // decoded symbols, same boxes
};

// One group of a full 32-lane group: lookup, state update, refill; returns
// the decoded value (symbol + offset).  The escape ballot is taken beside the
// refill; a group with an escape goes down the lane-serial path.
template <class F, bool SEARCH>
__device__ __forceinline__ int32_t dec_group_val(WarpDec<F> &st, const RowMeta &m,
                                                 const uint16_t *starts, const uint32_t *slots,
                                                 const typename F::Word *words, uint64_t nw,
                                                 uint32_t sh) {
  const int lane = threadIdx.x & 31;
  const uint32_t cum = F::cum16(st.x, sh);
  const uint32_t sym = lookup<SEARCH, true>(cum, m, starts, slots, true);
  const uint32_t start = starts[m.bucket_base + sym];
  const uint32_t freq = width_of(start, starts[m.bucket_base + sym + 1]);
  const typename F::State x = F::dec_step(st.x, cum, start, freq, sh);
  const bool esc = sym == m.maxv;
  const bool need = x < F::kLow;
  const uint32_t src = (uint32_t)lane >= st.off ? st.w0 : st.w1;
  const uint32_t nm = __ballot_sync(kFull, need);
  const bool any_esc = __any_sync(kFull, esc);
  const uint32_t j = st.off + __popc(nm & lanemask_lt());
  const uint32_t wv = __shfl_sync(kFull, src, j & 31);
  int32_t val = (int32_t)sym + m.offset;
  if (!any_esc) {
    st.x = need ? ((x << F::kWordBits) | wv) : x;
    st.off += __popc(nm);
    if (st.off >= 32) {
      st.w0 = st.w1;
      st.w1 = st.w2;
      st.cur += 32;
      st.off -= 32;
      st.w2 = word_at(words, nw, st.cur + 64 + lane);
    }
  } else {
    const EscapeResult<F> er = escape_group<F>(x, true, esc, m.maxv, st.cur + st.off, words, nw);
    st.x = er.x;
    if (esc) val = (int32_t)(er.val + (int64_t)m.offset);
    st.bad |= er.bad;
    st.cur = er.cur;
    st.off = 0;
    load_window(st, words, nw);
  }
  return val;
}

// Where a tiled stream's chunks are: the tensor-tile coordinates (x = first
// column, y = row, z = image * C + channel) of its next chunk, stepped 4 rows
// at a time through the tile and then to the next channel.
struct ChunkPos {
  int32_t y, z, y0, y1;  // y1 = y0 + tile height
  __device__ __forceinline__ void next() {
    y += 4;
    if (y == y1) {
      y = y0;
      ++z;
    }
  }
};

// Decodes stream s with tile staging; false when a bounded wait gave up (the
// warp then stops, its copies drained).
template <class F, bool SEARCH>
__device__ __forceinline__ bool decode_tile_stream(const DecCtx &c, const TileMaps &maps,
                                                   const RowMeta *meta, const uint16_t *starts,
                                                   const uint32_t *slots, uint32_t ring,
                                                   int32_t *ring_p, uint32_t bar0,
                                                   uint32_t &par, int64_t s) {
  using State = typename F::State;
  using Word = typename F::Word;
  const int lane = threadIdx.x & 31;
  const Geom &g = c.g;
  const StreamDesc d = stream_desc(g, s);
  const Word *words = nullptr;
  uint64_t nw = 0;
  if (!d.ok || !stream_bounds<F>(c, s, 32, words, nw)) {
    if (lane == 0) report(c.status, d.ok ? RANS_ERR_CORRUPT : RANS_ERR_ARG, s);
    return true;
  }
  if (lane == 0)
    bulk_prefetch_l2(reinterpret_cast<const char *>(c.in),
                     reinterpret_cast<const char *>(c.in) + c.in_bytes,
                     reinterpret_cast<const char *>(words + 64), sizeof(Word) * (nw - 64));
  const uint32_t sh = F::shift(c.sh);
  const uint32_t kmax = (uint32_t)c.K - 1u;
  // the tile: image b, channel group gi, tile row ty, tile column tx
  const int64_t per_img = g.ng * g.nty * g.ntx;
  const int64_t b = s / per_img, r0 = s - b * per_img;
  const int64_t gi = r0 / (g.nty * g.ntx), r1 = r0 - gi * (g.nty * g.ntx);
  const int64_t ty = r1 / g.ntx, tx = r1 - ty * g.ntx;
  const int32_t x0 = (int32_t)(tx * g.tw);
  const int32_t ww = d.t.ww, hh = d.t.hh;
  const int cls = ww == (int32_t)g.tw ? 0 : 1;
  const void *imap = &maps.idx[cls];
  const void *omap = &maps.out[cls];
  const int32_t Gc = ww >> 3;              // groups per chunk: 4 rows x ww / 32
  const uint32_t cbytes = 16u * (uint32_t)ww;
  const int32_t M = (int32_t)(d.n / (4 * ww));
  ChunkPos ld, sd;
  ld.y0 = ld.y = (int32_t)(ty * g.th);
  ld.y1 = ld.y0 + hh;
  ld.z = (int32_t)(b * g.C + gi * g.cg);
  sd = ld;
  ChunkPos pf = ld;  // the next chunk to prefetch into L2
  const uint32_t bar1 = bar0 + 8;
  // chunk 0 into half 0, once earlier stores have read the ring; chunks 1
  // and 2 into L2
  __syncwarp();
  if (lane == 0) {
    tma::bulk_wait_read();
    tma::fence_proxy_async();
    tma::arrive_expect(bar0, cbytes);
    tma::load_3d(ring, imap, x0, ld.y, ld.z, bar0);
  }
  ld.next();
  pf.next();
  for (int32_t q = 1; q < 3 && q < M; ++q) {
    if (lane == 0) tma::prefetch_l2_3d(imap, x0, pf.y, pf.z);
    pf.next();
  }
  const int32_t jload = Gc > 3 ? Gc - 3 : 0;  // the group after which chunk k + 1 loads

  WarpDec<F> st;
  st.x = (State)__ldg(words + 2 * lane) | ((State)__ldg(words + 2 * lane + 1) << F::kWordBits);
  st.cur = 64;
  st.off = 0;
  load_window(st, words, nw);
  st.rmax = 0;
  st.bad = false;
  auto meta_of = [&](uint32_t r) -> RowMeta {
    st.rmax = max(st.rmax, r);
    return row_meta(meta, min(r, kmax));
  };
  // loads in flight, by half (bit h)
  uint32_t pending = 1u;
  // a bounded wait for the chunk in half h; on giving up, a bounded wait for
  // every load still in flight, and the warp stops
  auto wait_half = [&](int h) -> bool {
    const uint32_t bar = h ? bar1 : bar0;
    const bool ok = tma::wait_bounded(bar, (par >> h) & 1u, kTileWaitTries);
    if (__all_sync(kFull, ok)) {
      par ^= 1u << h;
      pending &= ~(1u << h);
      return true;
    }
    if (lane == 0) report(c.status, RANS_ERR_TIMEOUT, s);
    for (int q = 0; q < 2; ++q)
      if (pending >> q & 1u) tma::wait_bounded(q ? bar1 : bar0, (par >> q) & 1u, kTileWaitTries);
    return false;
  };
  if (!wait_half(0)) return false;
  RowMeta m = meta_of((uint32_t)ring_p[lane]);
#pragma unroll 1
  for (int32_t k = 0; k < M; ++k) {
    const int h = k & 1;
    int32_t *rh = ring_p + h * (int32_t)(kTileRingHalf / 4);
#pragma unroll 1
    for (int32_t j = 0; j < Gc; ++j) {
      uint32_t rn = 0;
      if (j + 1 < Gc) {
        rn = (uint32_t)rh[(j + 1) * 32 + lane];
      } else if (k + 1 < M) {
        if (!wait_half(h ^ 1)) return false;
        rn = (uint32_t)ring_p[(h ^ 1) * (int32_t)(kTileRingHalf / 4) + lane];
      }
      const RowMeta mn = meta_of(rn);
      rh[j * 32 + lane] = dec_group_val<F, SEARCH>(st, m, starts, slots, words, nw, sh);
      if (j == 0 && k + 3 < M) {
        if (lane == 0) tma::prefetch_l2_3d(imap, x0, pf.y, pf.z);
        pf.next();
      }
      if (j == jload && k + 1 < M) {
        // chunk k + 1 into the other half, once chunk k - 1's store has read
        // it
        __syncwarp();
        if (lane == 0) {
          const uint32_t bar = h ? bar0 : bar1;
          tma::bulk_wait_read();
          tma::fence_proxy_async();
          tma::arrive_expect(bar, cbytes);
          tma::load_3d(ring + (uint32_t)(h ^ 1) * kTileRingHalf, imap, x0, ld.y, ld.z, bar);
        }
        pending |= 1u << (h ^ 1);
        ld.next();
      }
      m = mn;
    }
    // chunk k's decoded values go out
    tma::fence_proxy_async();
    __syncwarp();
    if (lane == 0) {
      tma::store_3d(omap, x0, sd.y, sd.z, ring + (uint32_t)h * kTileRingHalf);
      tma::bulk_commit();
    }
    sd.next();
  }
  if (__any_sync(kFull, st.rmax > kmax)) {
    if (lane == 0) report(c.status, RANS_ERR_INDEX, s);
    return true;
  }
  const bool ok = !st.bad && st.x == F::kLow && st.cur + st.off == nw;
  if (!__all_sync(kFull, ok) && lane == 0) report(c.status, RANS_ERR_CORRUPT, s);
  return true;
}

// ------------------------------------------ unrolled chunks, no branches --
// The decoder's time per group follows its instruction count: the state
// chain leaves little independent work, and a group body cut into small
// blocks by branches (the escape test, the window advance, the chunk
// bookkeeping) keeps the compiler from overlapping what there is.  For tile
// widths of 56 and 64 (7 and 8 groups per chunk) a chunk is therefore decoded
// as one unrolled block: the copy-engine work is predicated on lane 0,
// escapes are only recorded, and the only branch left is the window
// advance (about once in seven groups; the 64-bit format's variant below
// reads its words from a shared-memory window and has none).  A chunk in
// which any lane met an escape is decoded again from its saved state on the
// lane-serial path (its row indexes reloaded, since the fast pass overwrote
// them with values); the fast pass after an escape runs on a wrong state but
// reads only inside the tables, the register window and the stream's words.

// One full group on the fast path: lookup, state update and refill with no
// branch; a lane whose symbol is the escape bucket only sets `esc`.
template <class F>
__device__ __forceinline__ int32_t dec_group_fast(WarpDec<F> &st, const RowMeta &m,
                                                  const uint16_t *starts, const uint32_t *slots,
                                                  const typename F::Word *words, uint64_t nw,
                                                  uint32_t sh, uint32_t &esc) {
  const int lane = threadIdx.x & 31;
  const uint32_t cum = F::cum16(st.x, sh);
  const uint32_t sym = lookup<false, true>(cum, m, starts, slots, true);
  const uint32_t start = starts[m.bucket_base + sym];
  const uint32_t freq = width_of(start, starts[m.bucket_base + sym + 1]);
  const typename F::State x = F::dec_step(st.x, cum, start, freq, sh);
  esc |= sym == m.maxv ? 1u : 0u;
  const bool need = x < F::kLow;
  const uint32_t src = (uint32_t)lane >= st.off ? st.w0 : st.w1;
  const uint32_t nm = __ballot_sync(kFull, need);
  const uint32_t wv = __shfl_sync(kFull, src, st.off + __popc(nm & lanemask_lt()));
  st.x = need ? ((x << F::kWordBits) | wv) : x;
  st.off += __popc(nm);
  // the window advances about once in seven groups: behind a branch, so that
  // no instruction of the other groups reads the register whose load is
  // still in flight
  if (st.off >= 32) {
    st.w0 = st.w1;
    st.w1 = st.w2;
    st.cur += 32;
    st.off -= 32;
    st.w2 = word_at(words, nw, st.cur + 64 + lane);
  }
  return (int32_t)sym + m.offset;
}


__device__ __forceinline__ void chunk_next_if(ChunkPos &p, bool on) {
  const int32_t y = p.y + 4;
  const bool wrap = y == p.y1;
  p.y = on ? (wrap ? p.y0 : y) : p.y;
  p.z += on && wrap ? 1 : 0;
}

template <class F, int GC>
__device__ __forceinline__ bool decode_tile_stream_fast(const DecCtx &c, const TileMaps &maps,
                                                        const RowMeta *meta,
                                                        const uint16_t *starts,
                                                        const uint32_t *slots, uint32_t ring,
                                                        int32_t *ring_p, uint32_t bar0,
                                                        uint32_t &par, int64_t s) {
  using State = typename F::State;
  using Word = typename F::Word;
  constexpr int kJload = 0;  // chunk k + 1 loads right after chunk k's first group
  constexpr int kHalfW = (int)(kTileRingHalf / 4);
  const int lane = threadIdx.x & 31;
  const Geom &g = c.g;
  const StreamDesc d = stream_desc(g, s);
  const Word *words = nullptr;
  uint64_t nw = 0;
  if (!d.ok || !stream_bounds<F>(c, s, 32, words, nw)) {
    if (lane == 0) report(c.status, d.ok ? RANS_ERR_CORRUPT : RANS_ERR_ARG, s);
    return true;
  }
  if (lane == 0)
    bulk_prefetch_l2(reinterpret_cast<const char *>(c.in),
                     reinterpret_cast<const char *>(c.in) + c.in_bytes,
                     reinterpret_cast<const char *>(words + 64), sizeof(Word) * (nw - 64));
  const uint32_t sh = F::shift(c.sh);
  const uint32_t kmax = (uint32_t)c.K - 1u;
  const int64_t per_img = g.ng * g.nty * g.ntx;
  const int64_t b = s / per_img, t0 = s - b * per_img;
  const int64_t gi = t0 / (g.nty * g.ntx), t1 = t0 - gi * (g.nty * g.ntx);
  const int64_t ty = t1 / g.ntx, tx = t1 - ty * g.ntx;
  const int32_t x0 = (int32_t)(tx * g.tw);
  const int32_t hh = d.t.hh;
  const int cls = d.t.ww == (int32_t)g.tw ? 0 : 1;
  const void *imap = &maps.idx[cls];
  const void *omap = &maps.out[cls];
  const uint32_t cbytes = 128u * GC;
  const int32_t M = (int32_t)(d.n / (32 * GC));
  ChunkPos ld, sd;
  ld.y0 = ld.y = (int32_t)(ty * g.th);
  ld.y1 = ld.y0 + hh;
  ld.z = (int32_t)(b * g.C + gi * g.cg);
  sd = ld;
  ChunkPos pf = ld;
  const uint32_t bar1 = bar0 + 8;
  const uint32_t l0 = lane == 0 ? 1u : 0u;
  __syncwarp();
  tma::bulk_wait_read_if(l0);
  tma::fence_proxy_async();
  tma::arrive_expect_if(l0, bar0, cbytes);
  tma::load_3d_if(l0, ring, imap, x0, ld.y, ld.z, bar0);
  ld.next();
  pf.next();
  for (int32_t q = 1; q < 3 && q < M; ++q) {
    tma::prefetch_l2_3d_if(l0, imap, x0, pf.y, pf.z);
    pf.next();
  }
  uint32_t pending = 1u;

  WarpDec<F> st;
  st.x = (State)__ldg(words + 2 * lane) | ((State)__ldg(words + 2 * lane + 1) << F::kWordBits);
  st.cur = 64;
  st.off = 0;
  load_window(st, words, nw);
  st.rmax = 0;
  st.bad = false;
  auto meta_of = [&](uint32_t r) -> RowMeta {
    st.rmax = max(st.rmax, r);
    return row_meta(meta, min(r, kmax));
  };
  auto wait_half = [&](int h) -> bool {
    const uint32_t bar = h ? bar1 : bar0;
    const bool ok = tma::wait_bounded(bar, (par >> h) & 1u, kTileWaitTries);
    if (__all_sync(kFull, ok)) {
      par ^= 1u << h;
      pending &= ~(1u << h);
      return true;
    }
    if (lane == 0) report(c.status, RANS_ERR_TIMEOUT, s);
    for (int q = 0; q < 2; ++q)
      if (pending >> q & 1u) tma::wait_bounded(q ? bar1 : bar0, (par >> q) & 1u, kTileWaitTries);
    return false;
  };
#pragma unroll 1
  for (int32_t k = 0; k < M; ++k) {
    const int h = k & 1;
    if (!wait_half(h)) return false;
    int32_t *rh = ring_p + h * kHalfW;
    const uint32_t more1 = k + 1 < M ? 1u : 0u, more3 = k + 3 < M ? 1u : 0u;
    const WarpDec<F> st0 = st;
    uint32_t esc = 0;
    RowMeta m = meta_of((uint32_t)rh[lane]);
#pragma unroll
    for (int j = 0; j < GC; ++j) {
      RowMeta mn = m;
      if (j + 1 < GC) mn = meta_of((uint32_t)rh[(j + 1) * 32 + lane]);
      rh[j * 32 + lane] = dec_group_fast<F>(st, m, starts, slots, words, nw, sh, esc);
      if (j == 0) {
        tma::prefetch_l2_3d_if(l0 & more3, imap, x0, pf.y, pf.z);
        chunk_next_if(pf, more3 != 0);
      }
      if (j == kJload) {
        // chunk k + 1 into the other half, once chunk k - 1's store has read it
        __syncwarp();
        const uint32_t bar = h ? bar0 : bar1;
        tma::bulk_wait_read_if(l0 & more1);
        tma::fence_proxy_async();
        tma::arrive_expect_if(l0 & more1, bar, cbytes);
        tma::load_3d_if(l0 & more1, ring + (uint32_t)(h ^ 1) * kTileRingHalf, imap, x0, ld.y,
                        ld.z, bar);
        pending |= more1 << (h ^ 1);
        chunk_next_if(ld, more1 != 0);
      }
      m = mn;
    }
    if (__any_sync(kFull, esc != 0)) {
      // an escape in this chunk: reload its row indexes and decode it again
      // from its saved state on the lane-serial path
      __syncwarp();
      const uint32_t bar = h ? bar1 : bar0;
      tma::fence_proxy_async();
      tma::arrive_expect_if(l0, bar, cbytes);
      tma::load_3d_if(l0, ring + (uint32_t)h * kTileRingHalf, imap, x0, sd.y, sd.z, bar);
      pending |= 1u << h;
      if (!wait_half(h)) return false;
      st = st0;
#pragma unroll 1
      for (int j = 0; j < GC; ++j) {
        const RowMeta mj = meta_of((uint32_t)rh[j * 32 + lane]);
        rh[j * 32 + lane] = dec_group_val<F, false>(st, mj, starts, slots, words, nw, sh);
      }
    }
    // chunk k's decoded values go out
    tma::fence_proxy_async();
    __syncwarp();
    tma::store_3d_commit_if(l0, omap, x0, sd.y, sd.z, ring + (uint32_t)h * kTileRingHalf);
    sd.next();
  }
  if (__any_sync(kFull, st.rmax > kmax)) {
    if (lane == 0) report(c.status, RANS_ERR_INDEX, s);
    return true;
  }
  const bool ok = !st.bad && st.x == F::kLow && st.cur + st.off == nw;
  if (!__all_sync(kFull, ok) && lane == 0) report(c.status, RANS_ERR_CORRUPT, s);
  return true;
}

// ------------------------------------------ 64-bit format, word window --
// The 64-bit format's unrolled chunks keep the stream's words in a ring of
// kWinWords words in shared memory, refilled with cp.async once per chunk
// in blocks of 32 (the blocks the reads have passed).  A group reads its
// refill word from the ring (one shared load at the lane's rank among the
// lanes that refill) and takes no branch, so a chunk of 7 or 8 groups is
// one block of straight-line code.  The decoded values stay in registers
// until the chunk ends, so no store to the ring orders the groups' table
// reads.
constexpr uint32_t kWinWords = 512;
constexpr uint32_t kWinBytes = 4 * kWinWords;
static_assert(kTileStreamBytes == kTileRingBytes + kWinBytes, "index ring + word window");

// The tile origin of stream s: first column x0 and the chunk position of
// its first chunk.
__device__ __forceinline__ void tile_origin(const Geom &g, const StreamDesc &d, int64_t s,
                                            int32_t &x0, ChunkPos &p) {
  const int64_t per_img = g.ng * g.nty * g.ntx;
  const int64_t b = s / per_img, t0 = s - b * per_img;
  const int64_t gi = t0 / (g.nty * g.ntx), t1 = t0 - gi * (g.nty * g.ntx);
  const int64_t ty = t1 / g.ntx, tx = t1 - ty * g.ntx;
  x0 = (int32_t)(tx * g.tw);
  p.y0 = p.y = (int32_t)(ty * g.th);
  p.y1 = p.y0 + d.t.hh;
  p.z = (int32_t)(b * g.C + gi * g.cg);
}

// One group: lookup, state update and refill, no branch; a lane whose
// symbol is the escape bucket only sets `esc`.  win: the stream's word
// ring (word i at win[i mod kWinWords]), rd: the next word to read.
// SEARCH: a table with slots that ran out of bitmap room; those slots take
// the general lookup's binary search (a branch, entered once per warp).
// BW: the bucket's start and width from its bucket word (start | (width -
// 1) << 16, one load) instead of two 16-bit starts.
template <bool SEARCH, bool BW = false>
__device__ __forceinline__ int32_t dec_group_win64(uint64_t &x, uint32_t &rd, const RowMeta &m,
                                                   const uint16_t *starts, const uint32_t *slots,
                                                   const uint32_t *win, uint32_t &esc,
                                                   const uint32_t *bwords = nullptr) {
  const uint32_t xl = (uint32_t)x, xh = (uint32_t)(x >> 32);
  const uint32_t cum = xl & 0xffffu;
  uint32_t sym;
  if constexpr (SEARCH) {
    sym = lookup<true, true>(cum, m, starts, slots, true);
  } else {
    const uint32_t sh = m.slot >> 27;
    const uint32_t i1 = (m.slot & 0x07ffffffu) + (cum >> sh);
    const uint32_t se = slots[i1];
    const uint32_t c = cum & ((1u << sh) - 1u);
    const uint32_t lo = se & 0xffffu;
    const uint32_t e1 = __byte_perm(se, 0u, 0x4442u), e2 = se >> 24;
    sym = lo + (c > e1 ? 1u : 0u) + (c > e2 ? 1u : 0u);
    const bool bm = e1 == 0xffu && e2 != 0xffu;
    const uint32_t i2 = bm ? (lo | ((se >> 8) & 0xff0000u)) + (c >> 4) : i1;
    const uint32_t ce = slots[i2];
    const uint32_t sym2 = (ce >> 16) + __popc(ce & ((2u << (c & 15u)) - 1u));
    sym = min(bm ? sym2 : sym, m.maxv);
  }
  esc |= sym == m.maxv ? 1u : 0u;
  const uint32_t a = m.bucket_base + sym;
  uint32_t s0, f;
  if constexpr (BW) {
    const uint32_t e = bwords[a];
    s0 = e & 0xffffu;
    f = (e >> 16) + 1u;
  } else {
    const uint32_t s1 = starts[a + 1];
    s0 = starts[a];
    f = (s1 - s0) + (s1 == 0u ? 65536u : 0u);
  }
  // x' = f (x >> 16) + cum - start in 32-bit halves; refill when x' < 2^31
  const uint32_t tl = __funnelshift_r(xl, xh, 16), th = xh >> 16;
  const uint64_t p = (uint64_t)f * tl + (uint64_t)(cum - s0);
  const uint32_t nl = (uint32_t)p, nh = (uint32_t)(p >> 32) + f * th;
  const bool need = __funnelshift_r(nl, nh, 31) == 0u;
  const uint32_t bal = __ballot_sync(kFull, need);
  const uint32_t wv = win[(rd + __popc(bal & lanemask_lt())) & (kWinWords - 1u)];
  x = ((uint64_t)(need ? nl : nh) << 32) | (need ? wv : nl);
  rd += __popc(bal);
  return (int32_t)sym + m.offset;
}

// Loads the blocks of 32 words the reads have passed (once they land, the
// ring holds words [ldn - kWinWords, ldn)) with the words that follow; one
// cp.async commit group per call, possibly empty.  Word indexes past the
// stream read its last word.
__device__ __forceinline__ void win_refill(uint32_t *win, const uint32_t *words, uint32_t nw,
                                           uint32_t rd, uint32_t &ldn) {
  const uint32_t lane = threadIdx.x & 31;
  const uint32_t end = (rd & ~31u) + kWinWords;
#pragma unroll 1
  for (; ldn < end; ldn += 32) {
    const uint32_t wi = ldn + lane;
    cp_async4(win + (wi & (kWinWords - 1u)), words + (wi < nw ? wi : nw - 1u));
  }
  cp_async_commit();
}

// Stream s (64-bit format, tile width 56 or 64: GC = 7 or 8 groups a chunk,
// fewer than 2^31 words) on the unrolled path.  FLT: float latents: the
// index tile holds the scales (each group's row is its scale's table row,
// from the scale table `stab` in shared memory) and the output tile the
// values float(symbol) + mean, the means read from global memory at the
// chunk's start (0 without means).
// FM: 0 int32 rows, 1 float latents with the scale table searched, 2 float
// latents with its rows read through `keys`.
template <int GC, int FM, bool SEARCH>
__device__ __forceinline__ bool decode_tile_win64(const DecCtx &c, const TileMaps &maps,
                                                  const RowMeta *meta, const uint16_t *starts,
                                                  const uint32_t *slots, uint32_t ring,
                                                  int32_t *ring_p, uint32_t bar0, uint32_t &par,
                                                  int64_t s, const StreamDesc &d,
                                                  const uint32_t *words, uint32_t nw,
                                                  const float *stab, const ScaleKeys &keys) {
  constexpr bool FLT = FM != 0;
  constexpr int kHalfW = (int)(kTileRingHalf / 4);
  constexpr uint32_t cbytes = 128u * GC;
  const int lane = threadIdx.x & 31;
  const Geom &g = c.g;
  const uint32_t kmax = (uint32_t)c.K - 1u;
  const int cls = d.t.ww == (int32_t)g.tw ? 0 : 1;
  const void *imap = &maps.idx[cls];
  const void *omap = &maps.out[cls];
  const int32_t M = (int32_t)(d.n / (32 * GC));
  const uint32_t l0 = lane == 0 ? 1u : 0u;
  const uint32_t bar1 = bar0 + 8;
  uint32_t *win = reinterpret_cast<uint32_t *>(ring_p + kTileRingBytes / 4);
  int32_t x0;
  ChunkPos ld;
  tile_origin(g, d, s, x0, ld);
  ChunkPos sd = ld, pf = ld;
  if (lane == 0)
    bulk_prefetch_l2(reinterpret_cast<const char *>(c.in),
                     reinterpret_cast<const char *>(c.in) + c.in_bytes,
                     reinterpret_cast<const char *>(words + 64), sizeof(uint32_t) * (nw - 64));
  // chunk 0 into half 0, once earlier stores have read the ring; chunks 1
  // and 2 into L2
  __syncwarp();
  tma::bulk_wait_read_if(l0);
  tma::fence_proxy_async();
  tma::arrive_expect_if(l0, bar0, cbytes);
  tma::load_3d_if(l0, ring, imap, x0, ld.y, ld.z, bar0);
  ld.next();
  pf.next();
  for (int32_t q = 1; q < 3 && q < M; ++q) {
    tma::prefetch_l2_3d_if(l0, imap, x0, pf.y, pf.z);
    pf.next();
  }
  uint32_t pending = 1u;

  uint64_t x = (uint64_t)__ldg(words + 2 * lane) | ((uint64_t)__ldg(words + 2 * lane + 1) << 32);
  uint32_t rd = 64, ldn = 64, rmax = 0;
  bool bad = false;
  auto meta_of = [&](uint32_t r) -> RowMeta {
    if (FM == 1) r = scale_row(bound_scale(__uint_as_float(r), c.bound), stab, c.K);
    if (FM == 2) r = keys.row(bound_scale(__uint_as_float(r), c.bound));
    rmax = max(rmax, r);
    return row_meta(meta, min(r, kmax));
  };
  // FLT: a decoded value out (float(v) + mean as its bits), else v
  auto out_of = [&](int32_t v, float mean) -> int32_t {
    return FLT ? __float_as_int((float)v + mean) : v;
  };
  // FLT: group j's lane reads the mean of element e = 32 j + lane of the
  // chunk, row e / ww, column e mod ww
  int32_t moff[GC];
  if (FLT) {
#pragma unroll
    for (int j = 0; j < GC; ++j) {
      const int e = j * 32 + lane, r = e / (8 * GC);
      moff[j] = r * (int32_t)g.Wd + (e - r * 8 * GC);
    }
  }
  // a bounded wait for the chunk in half h; on giving up, a bounded wait for
  // every load still in flight, and the warp stops
  auto wait_half = [&](int h) -> bool {
    const uint32_t bar = h ? bar1 : bar0;
    const bool ok = tma::wait_bounded(bar, (par >> h) & 1u, kTileWaitTries);
    if (__all_sync(kFull, ok)) {
      par ^= 1u << h;
      pending &= ~(1u << h);
      return true;
    }
    if (lane == 0) report(c.status, RANS_ERR_TIMEOUT, s);
    for (int q = 0; q < 2; ++q)
      if (pending >> q & 1u) tma::wait_bounded(q ? bar1 : bar0, (par >> q) & 1u, kTileWaitTries);
    cp_async_wait<0>();
    return false;
  };
#pragma unroll 1
  for (int32_t k = 0; k < M; ++k) {
    const int h = k & 1;
    // the word window: top up, then wait for the words this chunk can read
    // (at most 32 a group): the blocks loaded before this chunk hold them
    // unless the window was just restarted
    const bool ahead = rd + 32u * GC <= ldn;
    win_refill(win, words, nw, rd, ldn);
    if (ahead) cp_async_wait<1>(); else cp_async_wait<0>();
    if (!wait_half(h)) return false;
    __syncwarp();  // every lane's window words, before any lane reads them
    const uint32_t more1 = k + 1 < M ? 1u : 0u, more3 = k + 3 < M ? 1u : 0u;
    int32_t *rh = ring_p + h * kHalfW;
    const uint64_t xs = x;
    const uint32_t rds = rd;
    uint32_t esc = 0;
    int32_t val[GC];
    float mu[GC];
    if (FLT) {
#pragma unroll
      for (int j = 0; j < GC; ++j) mu[j] = 0.0f;
      if (c.fmean) {
        const float *mp = c.fmean + (((int64_t)sd.z * g.H + sd.y) * g.Wd + x0);
#pragma unroll
        for (int j = 0; j < GC; ++j) mu[j] = __ldg(mp + moff[j]);
      }
    }
    // every group's row metadata first: they do not depend on the state
    RowMeta ms[GC];
#pragma unroll
    for (int j = 0; j < GC; ++j) ms[j] = meta_of((uint32_t)rh[j * 32 + lane]);
#pragma unroll
    for (int j = 0; j < GC; ++j) {
      val[j] = dec_group_win64<SEARCH>(x, rd, ms[j], starts, slots, win, esc);
      if (j == 0) {
        // chunk k + 3 into L2; chunk k + 1 into the other half, once chunk
        // k - 1's store has read it
        tma::prefetch_l2_3d_if(l0 & more3, imap, x0, pf.y, pf.z);
        chunk_next_if(pf, more3 != 0);
        __syncwarp();
        const uint32_t bar = h ? bar0 : bar1;
        tma::bulk_wait_read_if(l0 & more1);
        tma::fence_proxy_async();
        tma::arrive_expect_if(l0 & more1, bar, cbytes);
        tma::load_3d_if(l0 & more1, ring + (uint32_t)(h ^ 1) * kTileRingHalf, imap, x0, ld.y,
                        ld.z, bar);
        pending |= more1 << (h ^ 1);
        chunk_next_if(ld, more1 != 0);
      }
    }
    if (!__any_sync(kFull, esc != 0)) {
#pragma unroll
      for (int j = 0; j < GC; ++j) rh[j * 32 + lane] = out_of(val[j], FLT ? mu[j] : 0.0f);
    } else {
      // an escape in this chunk: decode it again from its saved state on
      // the lane-serial path (its row indexes are still in the ring), then
      // restart the word window where that left off
      WarpDec<Rans64> w;
      w.x = xs;
      w.cur = rds;
      w.off = 0;
      w.rmax = 0;
      w.bad = false;
      load_window(w, words, nw);
#pragma unroll 1
      for (int j = 0; j < GC; ++j) {
        const RowMeta mj = meta_of((uint32_t)rh[j * 32 + lane]);
        float mean = 0.0f;
        if (FLT) {
#pragma unroll
          for (int q = 0; q < GC; ++q) mean = q == j ? mu[q] : mean;
        }
        rh[j * 32 + lane] = out_of(
            dec_group_val<Rans64, SEARCH>(w, mj, starts, slots, words, nw, Rans64::shift(c.sh)),
            mean);
      }
      bad = bad || w.bad;
      x = w.x;
      rd = (uint32_t)(w.cur + w.off);
      cp_async_wait<0>();
      __syncwarp();
      ldn = rd & ~31u;
    }
    // chunk k's decoded values go out
    tma::fence_proxy_async();
    __syncwarp();
    tma::store_3d_commit_if(l0, omap, x0, sd.y, sd.z, ring + (uint32_t)h * kTileRingHalf);
    sd.next();
  }
  cp_async_wait<0>();
  if (__any_sync(kFull, rmax > kmax)) {
    if (lane == 0) report(c.status, RANS_ERR_INDEX, s);
    return true;
  }
  const bool ok = !bad && x == Rans64::kLow && rd == nw;
  if (!__all_sync(kFull, ok) && lane == 0) report(c.status, RANS_ERR_CORRUPT, s);
  return true;
}

// Stream s with the warp's ring and barriers: the unrolled chunks for tile
// widths 64 and 56 (8 and 7 groups) when its words are well formed and
// fewer than 2^31 (32-bit word cursors), the general loop otherwise or when
// the table has slots that search.
// FLT (float latents, 64-bit format): the unrolled path only (with the
// searching lookup when the table has slots that search); the host takes the
// tile kernel for them only when every tile is 64 or 56 wide, and a stream
// that is not well formed is reported here.
template <class F, bool FLT>
__device__ __forceinline__ bool decode_tile_one(const DecCtx &c, const TileMaps &maps,
                                                const RowMeta *meta, const uint16_t *starts,
                                                const uint32_t *slots, uint32_t ring,
                                                int32_t *ring_p, uint32_t bar0, uint32_t &par,
                                                int64_t s, bool search, const float *stab,
                                                const ScaleKeys &keys, bool use_keys) {
  const int lane = threadIdx.x & 31;
  if constexpr (!FLT) {
    if (search)
      return decode_tile_stream<F, true>(c, maps, meta, starts, slots, ring, ring_p, bar0, par,
                                         s);
  }
  const StreamDesc d = stream_desc(c.g, s);
  const typename F::Word *words = nullptr;
  uint64_t nw = 0;
  const bool fast = d.ok && (d.t.ww == 64 || d.t.ww == 56) &&
                    stream_bounds<F>(c, s, 32, words, nw) && nw < (uint64_t(1) << 31);
  if constexpr (FLT) {
    if (!fast) {
      if (lane == 0) report(c.status, d.ok ? RANS_ERR_CORRUPT : RANS_ERR_ARG, s);
      return true;
    }
  }
  if (fast) {
    if constexpr (std::is_same<F, Rans64>::value) {
      const uint32_t n32 = (uint32_t)nw;
      if constexpr (FLT) {
        const bool w64 = d.t.ww == 64;
        if (search && use_keys)
          return w64 ? decode_tile_win64<8, 2, true>(c, maps, meta, starts, slots, ring, ring_p, bar0, par, s, d, words, n32, stab, keys)
                     : decode_tile_win64<7, 2, true>(c, maps, meta, starts, slots, ring, ring_p, bar0, par, s, d, words, n32, stab, keys);
        if (search)
          return w64 ? decode_tile_win64<8, 1, true>(c, maps, meta, starts, slots, ring, ring_p, bar0, par, s, d, words, n32, stab, keys)
                     : decode_tile_win64<7, 1, true>(c, maps, meta, starts, slots, ring, ring_p, bar0, par, s, d, words, n32, stab, keys);
        if (use_keys)
          return w64 ? decode_tile_win64<8, 2, false>(c, maps, meta, starts, slots, ring, ring_p, bar0, par, s, d, words, n32, stab, keys)
                     : decode_tile_win64<7, 2, false>(c, maps, meta, starts, slots, ring, ring_p, bar0, par, s, d, words, n32, stab, keys);
        return w64 ? decode_tile_win64<8, 1, false>(c, maps, meta, starts, slots, ring, ring_p, bar0, par, s, d, words, n32, stab, keys)
                   : decode_tile_win64<7, 1, false>(c, maps, meta, starts, slots, ring, ring_p, bar0, par, s, d, words, n32, stab, keys);
      } else {
        if (d.t.ww == 64)
          return decode_tile_win64<8, 0, false>(c, maps, meta, starts, slots, ring, ring_p, bar0,
                                                par, s, d, words, n32, stab, keys);
        return decode_tile_win64<7, 0, false>(c, maps, meta, starts, slots, ring, ring_p, bar0,
                                              par, s, d, words, n32, stab, keys);
      }
    } else {
      if (d.t.ww == 64)
        return decode_tile_stream_fast<F, 8>(c, maps, meta, starts, slots, ring, ring_p, bar0,
                                             par, s);
      return decode_tile_stream_fast<F, 7>(c, maps, meta, starts, slots, ring, ring_p, bar0, par,
                                           s);
    }
  }
  if constexpr (!FLT)
    return decode_tile_stream<F, false>(c, maps, meta, starts, slots, ring, ring_p, bar0, par, s);
  return true;
}

// The tile-staged decoder: one stream per warp at a time, in scheduling
// order (largest tiles first).  FLT: float latents (scales in, values out).
template <class F, bool FLT>
__global__ void __launch_bounds__(kTileMaxStreams * 32, 1)
    decode_tile_kernel(DecCtx c, const __grid_constant__ TileMaps maps) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ uint64_t bar;
  __shared__ uint64_t ring_bar[kTileMaxStreams][2];
  const char *gb = c.blob + kHeaderBytes;
  if (!stage_to_smem(smem, gb, c.meta_bytes, &bar, c.status, smem + c.meta_bytes,
                     gb + c.meta_bytes + c.bucket_bytes, c.start_bytes + c.slot_bytes))
    return;
  const RowMeta *meta = reinterpret_cast<const RowMeta *>(smem);
  const uint16_t *starts = reinterpret_cast<const uint16_t *>(smem + c.meta_bytes);
  const uint32_t *slots = reinterpret_cast<const uint32_t *>(smem + c.meta_bytes + c.start_bytes);
  const uint32_t tab = c.meta_bytes + c.start_bytes + c.slot_bytes;
  const int warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5, lane = threadIdx.x & 31;
  // each warp's index ring and word window: 128-byte aligned (tensor-tile
  // copies)
  const uint32_t sbase = smem_addr(smem);
  const uint32_t ring = ((sbase + tab + 127u) & ~127u) + (uint32_t)warp * kTileStreamBytes;
  int32_t *ring_p = reinterpret_cast<int32_t *>(smem + (ring - sbase));
  const uint32_t bar0 = smem_addr(&ring_bar[warp][0]);
  // FLT: the scale table after every warp's ring, then its key counts
  float *stab = nullptr;
  ScaleKeys keys{};
  bool use_keys = false;
  if (FLT) {
    stab = reinterpret_cast<float *>(smem + (((sbase + tab + 127u) & ~127u) - sbase) +
                                     (uint32_t)nwarp * kTileStreamBytes);
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
  // slots that ran out of bitmap room (flagged in the blob header) search
  const bool search = reinterpret_cast<const uint32_t *>(c.blob)[kSearchFlagWord] != 0;
  for (int64_t k = blockIdx.x + (int64_t)gridDim.x * warp; k < c.g.S;
       k += (int64_t)gridDim.x * nwarp) {
    if (!decode_tile_one<F, FLT>(c, maps, meta, starts, slots, ring, ring_p, bar0, par,
                                 stream_of(c.g, k), search, stab, keys, use_keys))
      break;
  }
  if (lane == 0) tma::bulk_wait_all();
}

// --------------------------------------------- contiguous chunked streams --
// Contiguous streams (64-bit format, W = 32) made of whole chunks of 256
// symbols whose row changes at most once per chunk (an index block of 256
// symbols or more; the byte sweep's shape): a chunk's row index is one load,
// read a chunk ahead, and its metadata one shared load; its 8 groups decode
// as one block of straight-line code on the shared-memory word window; its
// values go to a two-half ring in shared memory and out with one bulk store.
constexpr int kChunkSyms = 256;

// PER: one row index per symbol, staged through a two-half ring with the
// chunk's values (else one per chunk, read directly).
template <typename SymT, bool PER>
__host__ __device__ constexpr uint32_t chunk_warp_bytes() {
  return kWinBytes + 2u * (uint32_t)kChunkSyms * (uint32_t)sizeof(SymT) +
         (PER ? 2u * (uint32_t)kChunkSyms * 4u : 0u);
}

template <typename SymT, bool SEARCH, bool PER, bool BW = false>
__device__ __forceinline__ void decode_chunk_stream(const DecCtx &c, const RowMeta *meta,
                                                    const uint16_t *starts,
                                                    const uint32_t *slots, uint32_t *win,
                                                    SymT *oring, int32_t *iring, int64_t s,
                                                    const uint32_t *bwords = nullptr) {
  constexpr int GC = kChunkSyms / 32;
  const int lane = threadIdx.x & 31;
  const Geom &g = c.g;
  const StreamDesc d = stream_desc(g, s);
  const uint32_t *words = nullptr;
  uint64_t nw64 = 0;
  if (!d.ok || !stream_bounds<Rans64>(c, s, 32, words, nw64) || nw64 >= (uint64_t(1) << 31)) {
    if (lane == 0) report(c.status, d.ok ? RANS_ERR_CORRUPT : RANS_ERR_ARG, s);
    return;
  }
  const uint32_t nw = (uint32_t)nw64;
  const uint32_t kmax = (uint32_t)c.K - 1u;
  const int32_t M = (int32_t)(d.n / kChunkSyms);
  const int ib = g.ib_shift;
  const uint32_t l0 = lane == 0 ? 1u : 0u;
  SymT *out = reinterpret_cast<SymT *>(c.out) + d.base;
  if (lane == 0)
    bulk_prefetch_l2(reinterpret_cast<const char *>(c.in),
                     reinterpret_cast<const char *>(c.in) + c.in_bytes,
                     reinterpret_cast<const char *>(words + 64), sizeof(uint32_t) * (nw - 64));
  uint64_t x = (uint64_t)__ldg(words + 2 * lane) | ((uint64_t)__ldg(words + 2 * lane + 1) << 32);
  uint32_t rd = 64, ldn = 64, rmax = 0;
  bool bad = false;
  // PER: chunk k's row indexes into index ring half k & 1 (16-byte copies,
  // one commit group per call, possibly empty)
  auto rows_in = [&](int32_t k) {
    if (k < M) {
      const int32_t *src = c.idx + d.base + (int64_t)k * kChunkSyms;
      int32_t *dst = iring + (k & 1) * kChunkSyms;
#pragma unroll
      for (int o = lane * 4; o < kChunkSyms; o += 128) cp_async16(dst + o, src + o);
    }
    cp_async_commit();
  };
  if (PER) rows_in(0);
  uint32_t r_next = PER ? 0u : (uint32_t)__ldg(c.idx + (d.base >> ib));
#pragma unroll 1
  for (int32_t k = 0; k < M; ++k) {
    const int h = k & 1;
    RowMeta ms[GC];
    if (!PER) {
      const uint32_t r = r_next;
      if (k + 1 < M)
        r_next = (uint32_t)__ldg(c.idx + ((d.base + (int64_t)(k + 1) * kChunkSyms) >> ib));
      rmax = max(rmax, r);
      const RowMeta m = row_meta(meta, min(r, kmax));
#pragma unroll
      for (int j = 0; j < GC; ++j) ms[j] = m;
    }
    // PER: chunk k + 1's rows on their way; the word window (as the tile
    // decoder's); then the rows of chunk k and the blocks read before this
    // chunk have landed (the two newest commit groups may still be in flight)
    if (PER) rows_in(k + 1);
    const bool ahead = rd + 32u * GC <= ldn;
    win_refill(win, words, nw, rd, ldn);
    if (ahead) {
      if (PER) cp_async_wait<2>(); else cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    // the ring half of this chunk's values, once chunk k - 2's store has read
    // it
    tma::bulk_wait_read1_if(l0);
    __syncwarp();
    if (PER) {
      const int32_t *rk = iring + h * kChunkSyms;
#pragma unroll
      for (int j = 0; j < GC; ++j) {
        const uint32_t r = (uint32_t)rk[j * 32 + lane];
        rmax = max(rmax, r);
        ms[j] = row_meta(meta, min(r, kmax));
      }
    }
    const uint64_t xs = x;
    const uint32_t rds = rd;
    uint32_t esc = 0;
    int32_t val[GC];
#pragma unroll
    for (int j = 0; j < GC; ++j)
      val[j] = dec_group_win64<SEARCH, BW>(x, rd, ms[j], starts, slots, win, esc, bwords);
    SymT *oh = oring + h * kChunkSyms;
    if (!__any_sync(kFull, esc != 0)) {
#pragma unroll
      for (int j = 0; j < GC; ++j) oh[j * 32 + lane] = (SymT)val[j];
    } else {
      // an escape in this chunk: decode it again from its saved state on
      // the lane-serial path, then restart the word window there
      WarpDec<Rans64> w;
      w.x = xs;
      w.cur = rds;
      w.off = 0;
      w.rmax = 0;
      w.bad = false;
      load_window(w, words, nw);
#pragma unroll 1
      for (int j = 0; j < GC; ++j) {
        RowMeta mj = ms[0];
#pragma unroll
        for (int q = 1; q < GC; ++q) mj = q == j ? ms[q] : mj;
        oh[j * 32 + lane] =
            (SymT)dec_group_val<Rans64, SEARCH>(w, mj, starts, slots, words, nw, 0u);
      }
      bad = bad || w.bad;
      x = w.x;
      rd = (uint32_t)(w.cur + w.off);
      cp_async_wait<0>();
      __syncwarp();
      ldn = rd & ~31u;
    }
    // the chunk's values go out
    tma::fence_proxy_async();
    __syncwarp();
    tma::store_1d_commit_if(l0, out + (int64_t)k * kChunkSyms, smem_addr(oh),
                            (uint32_t)(kChunkSyms * sizeof(SymT)));
  }
  cp_async_wait<0>();
  if (__any_sync(kFull, rmax > kmax)) {
    if (lane == 0) report(c.status, RANS_ERR_INDEX, s);
    return;
  }
  const bool ok = !bad && x == Rans64::kLow && rd == nw;
  if (!__all_sync(kFull, ok) && lane == 0) report(c.status, RANS_ERR_CORRUPT, s);
}

constexpr int kChunkMaxWarps = 32;  // a 2^28-symbol sweep's 8,192 streams in two rounds

// (per-symbol rows: at most 16 warps, so that the chunk's eight row
// metadata fit in registers)
constexpr int kChunkPerMaxWarps = 16;

// BW: the bucket words are staged too (the blob's meta, bucket words,
// starts and slots in one range) and the fast path reads them.
template <typename SymT, bool PER, bool BW = false>
__global__ void __launch_bounds__((PER ? kChunkPerMaxWarps : kChunkMaxWarps) * 32, 1)
    decode_chunk_kernel(DecCtx c) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ uint64_t bar;
  const char *gb = c.blob + kHeaderBytes;
  const uint32_t bwb = BW ? c.bucket_bytes : 0u;  // staged bucket-word bytes
  if (BW) {
    if (!stage_to_smem(smem, gb, c.meta_bytes + c.bucket_bytes + c.start_bytes + c.slot_bytes,
                       &bar, c.status))
      return;
  } else {
    if (!stage_to_smem(smem, gb, c.meta_bytes, &bar, c.status, smem + c.meta_bytes,
                       gb + c.meta_bytes + c.bucket_bytes, c.start_bytes + c.slot_bytes))
      return;
  }
  const RowMeta *meta = reinterpret_cast<const RowMeta *>(smem);
  const uint32_t *bwords = BW ? reinterpret_cast<const uint32_t *>(smem + c.meta_bytes) : nullptr;
  const uint16_t *starts = reinterpret_cast<const uint16_t *>(smem + c.meta_bytes + bwb);
  const uint32_t *slots =
      reinterpret_cast<const uint32_t *>(smem + c.meta_bytes + bwb + c.start_bytes);
  const uint32_t tab = c.meta_bytes + bwb + c.start_bytes + c.slot_bytes;
  const int warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
  // each warp's word window and value ring, 128-byte aligned
  const uint32_t sbase = smem_addr(smem);
  const uint32_t wbase =
      ((sbase + tab + 127u) & ~127u) + (uint32_t)warp * chunk_warp_bytes<SymT, PER>();
  uint32_t *win = reinterpret_cast<uint32_t *>(smem + (wbase - sbase));
  SymT *oring = reinterpret_cast<SymT *>(smem + (wbase - sbase) + kWinBytes);
  int32_t *iring = reinterpret_cast<int32_t *>(smem + (wbase - sbase) + kWinBytes +
                                               2u * kChunkSyms * sizeof(SymT));
  // slots that ran out of bitmap room (flagged in the blob header) search
  const bool search = reinterpret_cast<const uint32_t *>(c.blob)[kSearchFlagWord] != 0;
  for (int64_t k = blockIdx.x + (int64_t)gridDim.x * warp; k < c.g.S;
       k += (int64_t)gridDim.x * nwarp) {
    if (search)
      decode_chunk_stream<SymT, true, PER, BW>(c, meta, starts, slots, win, oring, iring, k,
                                               bwords);
    else
      decode_chunk_stream<SymT, false, PER, BW>(c, meta, starts, slots, win, oring, iring, k,
                                                bwords);
  }
  if ((threadIdx.x & 31) == 0) tma::bulk_wait_all();
}

// Whether a tiled W = 32 decode can take the tile-staged kernel: int32 rows
// and symbols in 16-byte aligned tensors, one index per element, every tile
// row a whole number of 16-byte units and of 8-symbol steps (so a chunk of 4
// rows is a whole number of groups, at least 2), tile heights multiples of 4,
// and the row metadata, starts, slots and rings in shared memory.
bool tile_path_ok(const DecCtx &c, int mode, int sym_dtype, const void *indexes,
                  const void *symbols) {
  const Geom &g = c.g;
  if (g.kind != RANS_CHUNK_TILED || g.W != 32 || g.alias || mode != 1 || g.ib_shift != 0 ||
      sym_dtype != RANS_SYM_INT32)
    return false;
  if ((reinterpret_cast<uintptr_t>(indexes) & 15) || (reinterpret_cast<uintptr_t>(symbols) & 15))
    return false;
  const int64_t ww1 = g.Wd % g.tw, hh1 = g.H % g.th;
  auto width_ok = [](int64_t w) { return w % 8 == 0 && w >= 16 && w <= 64; };
  if (!width_ok(g.tw > g.Wd ? g.Wd : g.tw) || (ww1 != 0 && !width_ok(ww1))) return false;
  if (g.th % 4 != 0 || hh1 % 4 != 0 || g.Wd % 4 != 0) return false;
  return true;
}

// Launches the tile-staged decoder; kNotTaken when the tables and rings do
// not fit in shared memory (the caller then takes the general kernel).
constexpr int kNotTaken = 1;

template <class F, bool FLT = false>
int launch_decode_tile(const DecCtx &c, const void *indexes, void *symbols, cudaStream_t st) {
  const Geom &g = c.g;
  int dev = 0;
  cudaGetDevice(&dev);
  const uint32_t tab = dec_table_bytes(1, c);
  const uint32_t stab_bytes =
      FLT ? (uint32_t)pad16(4ull * (uint64_t)c.K) + kScaleKeyBytes : 0u;
  const int optin = smem_optin(dev);
  const uint32_t lim = (uint32_t)optin - 64u - 2u * 8u * kTileMaxStreams - stab_bytes;
  if (tab + 128u + kTileStreamBytes > lim) return kNotTaken;
  TileMaps maps;
  const int64_t per_img = g.ng * g.nty * g.ntx;
  const int64_t depth = (g.S / per_img) * g.C;
  const uint32_t w0 = (uint32_t)(g.tw > g.Wd ? g.Wd : g.tw);
  const uint32_t w1 = g.Wd % g.tw ? (uint32_t)(g.Wd % g.tw) : w0;
  for (int k = 0; k < 2; ++k) {
    const uint32_t bw = k ? w1 : w0;
    if (encode_tile_map(&maps.idx[k], indexes, g.Wd, g.H, depth, bw, 4) ||
        encode_tile_map(&maps.out[k], symbols, g.Wd, g.H, depth, bw, 4))
      return RANS_ERR_CUDA;
  }
  const int sms = num_sms(dev);
  int64_t warps = (g.S + sms - 1) / sms;
  if (warps > kTileMaxStreams) warps = kTileMaxStreams;
  const int64_t room = ((int64_t)lim - tab - 128) / kTileStreamBytes;
  if (warps > room) warps = room;
  if (warps < 1) warps = 1;
  const uint32_t smem = tab + 128u + (uint32_t)warps * kTileStreamBytes + stab_bytes;
  auto kern = decode_tile_kernel<F, FLT>;
  if (ensure_dyn_smem((const void *)kern, smem) != cudaSuccess) return RANS_ERR_CUDA;
  int fit = 0;
  if (blocks_per_sm(&fit, (const void *)kern, (int)warps * 32, smem) != cudaSuccess || fit < 1)
    return RANS_ERR_CUDA;
  const int64_t need = (g.S + warps - 1) / warps;
  const int64_t cap = (int64_t)fit * sms;
  const int64_t blocks = need < cap ? need : cap;
  kern<<<(unsigned)blocks, (unsigned)warps * 32, smem, st>>>(c, maps);
  return cudaGetLastError() == cudaSuccess ? RANS_OK : RANS_ERR_CUDA;
}

// Whether a decode can take the chunked kernel: contiguous W = 32 streams of
// the 64-bit format, every stream a whole number of 256-symbol chunks, an
// index block of at least 256 symbols, the tables' lookup slots in shared
// memory, and a 16-byte aligned output of 1-, 2- or 4-byte symbols.
bool chunk_path_ok(const DecCtx &c, int mode, int sym_dtype, const void *symbols) {
  const Geom &g = c.g;
  if (g.kind != RANS_CHUNK_CONTIG || g.W != 32 || g.alias || g.fmt != RANS_FMT_RANS64 ||
      mode != 1 || (g.ib_shift != 0 && g.ib_shift < 8))
    return false;
  if (g.ib_shift == 0 && (reinterpret_cast<uintptr_t>(c.idx) & 15) != 0) return false;
  if (sym_dtype != RANS_SYM_UINT8 && sym_dtype != RANS_SYM_INT16 && sym_dtype != RANS_SYM_INT32)
    return false;
  if (g.per < kChunkSyms || g.per % kChunkSyms != 0 || g.per > (int64_t(1) << 28) ||
      g.n != g.S * g.per)
    return false;
  return (reinterpret_cast<uintptr_t>(symbols) & 15) == 0;
}

template <typename SymT, bool PER>
int launch_decode_chunk(const DecCtx &c, cudaStream_t st) {
  const Geom &g = c.g;
  int dev = 0;
  cudaGetDevice(&dev);
  const uint32_t tab = dec_table_bytes(1, c);
  const uint32_t per_warp = chunk_warp_bytes<SymT, PER>();
  const uint32_t lim = (uint32_t)smem_optin(dev) - 64u;
  if (tab + 128u + per_warp > lim) return kNotTaken;
  const int sms = num_sms(dev);
  int64_t warps = (g.S + sms - 1) / sms;
  const int64_t max_warps = PER ? kChunkPerMaxWarps : kChunkMaxWarps;
  if (warps > max_warps) warps = max_warps;
  // the bucket words staged as well when that costs no warps
  const bool bw = (int64_t)tab + c.bucket_bytes + 128 + warps * per_warp <= (int64_t)lim;
  const uint32_t tabw = tab + (bw ? c.bucket_bytes : 0u);
  const int64_t room = ((int64_t)lim - tabw - 128) / per_warp;
  if (warps > room) warps = room;
  if (warps < 1) warps = 1;
  const uint32_t smem = tabw + 128u + (uint32_t)warps * per_warp;
  auto kern = bw ? decode_chunk_kernel<SymT, PER, true> : decode_chunk_kernel<SymT, PER>;
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

template <class F, int W, typename SymT, int MODE, bool IB0>
__global__ void __launch_bounds__(W == 32 ? kDecMaxThreads32 : kDecThreads1)
    decode_kernel(DecCtx c) {
  constexpr bool ROWS = MODE == 2;
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ uint64_t bar;
  const RowMeta *meta;
  const uint16_t *buckets;  // 16-bit starts
  const uint32_t *slots;
  const char *gb = c.blob + kHeaderBytes;
  if (MODE != 0) {
    // [meta][starts]([slots]) in shared memory, from two ranges of the blob
    if (!stage_to_smem(smem, gb, c.meta_bytes, &bar, c.status, smem + c.meta_bytes,
                       gb + c.meta_bytes + c.bucket_bytes,
                       c.start_bytes + (MODE == 1 ? c.slot_bytes : 0u)))
      return;
    meta = reinterpret_cast<const RowMeta *>(smem);
    buckets = reinterpret_cast<const uint16_t *>(smem + c.meta_bytes);
    slots = reinterpret_cast<const uint32_t *>(smem + c.meta_bytes + c.start_bytes);
  } else {
    meta = reinterpret_cast<const RowMeta *>(gb);
    buckets = reinterpret_cast<const uint16_t *>(gb + c.meta_bytes + c.bucket_bytes);
    slots = reinterpret_cast<const uint32_t *>(gb + c.meta_bytes + c.bucket_bytes + c.start_bytes);
  }
  const uint32_t tab = dec_table_bytes(MODE, c);
  // float values: the scale table, copied after the stage rings when it fits
  const float *stab = c.stab;
  if (std::is_same<SymT, float>::value && c.stab_smem) {
    float *t = reinterpret_cast<float *>(
        smem + tab + (W == 32 ? (blockDim.x >> 5) * (uint32_t)(kDecStage * 32 * 4) : 0));
    for (int i = threadIdx.x; i < c.K; i += blockDim.x) t[i] = c.stab[i];
    __syncthreads();
    stab = t;
  }
  if (W == 32) {
    const int warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    uint32_t *stg = reinterpret_cast<uint32_t *>(smem + tab) + warp * kDecStage * 32;
    // slots that ran out of bitmap room (flagged in the blob header) search
    const bool search =
        !ROWS && reinterpret_cast<const uint32_t *>(c.blob)[kSearchFlagWord] != 0;
    for (int64_t k = blockIdx.x + (int64_t)gridDim.x * warp; k < c.g.S;
         k += (int64_t)gridDim.x * nw) {
      if (search)
        decode_stream_w32_entry<F, SymT, IB0, true, ROWS>(c, meta, buckets, slots, stg,
                                                          stream_of(c.g, k), stab);
      else
        decode_stream_w32_entry<F, SymT, IB0, false, ROWS>(c, meta, buckets, slots, stg,
                                                           stream_of(c.g, k), stab);
    }
  } else {
    // contiguous or explicit streams of integer symbols take the four-symbol
    // loop, tiled streams and float values the general one
    const bool flat = !std::is_same<SymT, float>::value && c.g.kind != RANS_CHUNK_TILED;
    for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < c.g.S;
         k += (int64_t)gridDim.x * blockDim.x) {
      if constexpr (!std::is_same<SymT, float>::value) {
        if (flat) {
          decode_stream_w1c<F, SymT, ROWS>(c, meta, buckets, slots, stream_of(c.g, k));
          continue;
        }
      }
      decode_stream_w1<F, SymT, ROWS>(c, meta, buckets, slots, stream_of(c.g, k), stab);
    }
  }
}

// W = 2, 4 or 8: 32 / W streams per warp (decode_segment); the table mode is
// a run-time argument.
constexpr int kSegThreads = 256;

template <class F, typename SymT, bool ALIAS>
__global__ void __launch_bounds__(kSegThreads) decode_kernel_wn(DecCtx c, int mode) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ uint64_t bar;
  const char *gb = c.blob + kHeaderBytes;
  const RowMeta *meta = reinterpret_cast<const RowMeta *>(gb);
  const uint16_t *buckets = reinterpret_cast<const uint16_t *>(gb + c.meta_bytes + c.bucket_bytes);
  const uint32_t *slots =
      reinterpret_cast<const uint32_t *>(gb + c.meta_bytes + c.bucket_bytes + c.start_bytes);
  if (mode != 0) {
    if (!stage_to_smem(smem, gb, c.meta_bytes, &bar, c.status, smem + c.meta_bytes,
                       gb + c.meta_bytes + c.bucket_bytes,
                       c.start_bytes + (mode == 1 ? c.slot_bytes : 0u)))
      return;
    meta = reinterpret_cast<const RowMeta *>(smem);
    buckets = reinterpret_cast<const uint16_t *>(smem + c.meta_bytes);
    slots = reinterpret_cast<const uint32_t *>(smem + c.meta_bytes + c.start_bytes);
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
      decode_segment<F, SymT, true, ALIAS>(c, meta, buckets, slots, s, W);
    else
      decode_segment<F, SymT, false, ALIAS>(c, meta, buckets, slots, s, W);
  }
}

template <class F, typename SymT, bool ALIAS>
int launch_decode_wn(const DecCtx &c, int mode, cudaStream_t st) {
  auto kern = decode_kernel_wn<F, SymT, ALIAS>;
  const uint32_t tab = dec_table_bytes(mode, c);
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

template <class F, int W, typename SymT, int MODE, bool IB0>
int launch_decode_t(const DecCtx &c, cudaStream_t st) {
  auto kern = decode_kernel<F, W, SymT, MODE, IB0>;
  const uint32_t tab = dec_table_bytes(MODE, c);
  const uint32_t per_warp = W == 32 ? kDecStage * 32 * 4 : 0;
  int dev = 0;
  cudaGetDevice(&dev);
  // float latents: the scale table goes after the stage rings when it fits
  const uint32_t tbl = std::is_same<SymT, float>::value ? (uint32_t)pad16(4ull * (uint64_t)c.K) : 0u;
  const int optin = smem_optin(dev);
  const uint32_t lim = (uint32_t)optin - 64u;  // room for the kernel's static shared memory
  const uint32_t max_dyn = tab + kDecStageBytes + tbl <= lim ? tab + kDecStageBytes + tbl : lim;
  if (ensure_dyn_smem((const void *)kern, (uint32_t)(max_dyn)) !=
      cudaSuccess)
    return RANS_ERR_CUDA;
  const int sms = num_sms(dev);
  int threads, blocks;
  uint32_t smem = tab;
  if (W == 32) {
    // One or a few CTAs per SM (bounded by the staged tables); enough warps
    // for one stream each when possible.
    int per_sm = 0;
    if (blocks_per_sm(&per_sm, (const void *)kern, 32, (uint32_t)(tab + per_warp)) !=
            cudaSuccess ||
        per_sm < 1)
      return RANS_ERR_CUDA;
    int64_t nblk = (int64_t)sms * per_sm;
    if (nblk > c.g.S) nblk = c.g.S < 1 ? 1 : c.g.S;
    int64_t warps = (c.g.S + nblk - 1) / nblk;
    if (warps > kDecMaxWarps) warps = kDecMaxWarps;
    if (warps < 1) warps = 1;
    threads = (int)warps * 32;
    smem = tab + (uint32_t)warps * per_warp;
    int fit = 0;
    if (blocks_per_sm(&fit, (const void *)kern, threads, (uint32_t)(smem)) != cudaSuccess ||
        fit < 1)
      return RANS_ERR_CUDA;
    int64_t need = (c.g.S + warps - 1) / warps;
    int64_t cap = (int64_t)fit * sms;
    blocks = (int)(need < cap ? need : cap);
  } else {
    threads = kDecThreads1;
    int fit = 0;
    if (blocks_per_sm(&fit, (const void *)kern, threads, (uint32_t)(smem)) != cudaSuccess ||
        fit < 1)
      return RANS_ERR_CUDA;
    int64_t need = (c.g.S + threads - 1) / threads;
    int64_t cap = (int64_t)fit * sms;
    blocks = (int)(need < cap ? need : cap);
  }
  if (blocks < 1) blocks = 1;
  DecCtx cc = c;
  cc.stab_smem = tbl > 0 && smem + tbl <= max_dyn ? 1 : 0;
  if (cc.stab_smem) smem += tbl;
  kern<<<blocks, threads, smem, st>>>(cc);
  return cudaGetLastError() == cudaSuccess ? RANS_OK : RANS_ERR_CUDA;
}

template <class F, int W, typename SymT, int MODE>
int launch_decode_m(const DecCtx &c, cudaStream_t st) {
  return c.g.ib_shift == 0 ? launch_decode_t<F, W, SymT, MODE, true>(c, st)
                           : launch_decode_t<F, W, SymT, MODE, false>(c, st);
}

template <class F, int W, typename SymT>
int launch_decode_w(const DecCtx &c, int mode, cudaStream_t st) {
  if (mode == 1) return launch_decode_m<F, W, SymT, 1>(c, st);
  if (mode == 2) return launch_decode_m<F, W, SymT, 2>(c, st);
  return launch_decode_m<F, W, SymT, 0>(c, st);
}

template <class F, typename SymT>
int launch_decode_f(const DecCtx &c, int mode, cudaStream_t st) {
  if (c.g.alias) return launch_decode_wn<F, SymT, true>(c, mode, st);  // W = 1, 2, 4, 8
  if (c.g.W == 32) return launch_decode_w<F, 32, SymT>(c, mode, st);
  if (c.g.W == 1) return launch_decode_w<F, 1, SymT>(c, mode, st);
  return launch_decode_wn<F, SymT, false>(c, mode, st);
}

template <typename SymT>
int launch_decode_s(const DecCtx &c, int mode, cudaStream_t st) {
  return c.g.fmt == RANS_FMT_RANS32_16 ? launch_decode_f<Rans32, SymT>(c, mode, st)
                                       : launch_decode_f<Rans64, SymT>(c, mode, st);
}

}  // namespace

int launch_decode_float(const uint8_t *in, uint64_t in_bytes, const uint64_t *offsets,
                        const float *scales, const float *means, const float *scale_table,
                        float scale_bound, const rans_tables &t, const Geom &g, float *values,
                        int32_t *status, cudaStream_t st) {
  DecCtx c;
  c.in = in;
  c.in_bytes = in_bytes;
  c.offs = offsets;
  c.idx = nullptr;
  c.K = t.K;
  c.sh = 0;
  c.aslots = nullptr;
  c.meta_bytes = t.meta_bytes;
  c.bucket_bytes = t.bucket_bytes;
  c.start_bytes = t.start_bytes;
  c.slot_bytes = t.slot_bytes;
  c.blob = reinterpret_cast<const char *>(t.blob);
  c.g = g;
  c.out = values;
  c.status = status;
  c.fscale = scales;
  c.fmean = means;
  c.stab = scale_table;
  c.bound = scale_bound;
  // float values decode the 64-bit format only (the caller checks); tiled
  // streams of 64- and 56-wide tiles take the tile-staged kernel (scales in
  // as the index tiles, values out as the symbol tiles)
  if (t.dec_in_smem == 1 && flt_tile_shape_ok(g, scales, values)) {
    const int r = launch_decode_tile<Rans64, true>(c, scales, values, st);
    if (r != kNotTaken) return r;
  }
  return g.W == 32 ? launch_decode_w<Rans64, 32, float>(c, t.dec_in_smem, st)
                   : launch_decode_w<Rans64, 1, float>(c, t.dec_in_smem, st);
}

int launch_decode(const uint8_t *in, uint64_t in_bytes, const uint64_t *offsets,
                  const int32_t *indexes, const rans_tables &t, const Geom &g, void *symbols,
                  int sym_dtype, int32_t *status, cudaStream_t st) {
  DecCtx c;
  c.in = in;
  c.in_bytes = in_bytes;
  c.offs = offsets;
  c.idx = indexes;
  c.K = t.K;
  c.sh = (uint32_t)(kPrec - t.precision);
  c.aslots = g.alias ? reinterpret_cast<const uint2 *>(t.alias) : nullptr;
  c.meta_bytes = t.meta_bytes;
  c.bucket_bytes = t.bucket_bytes;
  c.start_bytes = t.start_bytes;
  c.slot_bytes = t.slot_bytes;
  c.blob = reinterpret_cast<const char *>(t.blob);
  c.g = g;
  c.out = symbols;
  c.status = status;
  c.fscale = c.fmean = c.stab = nullptr;
  c.bound = 0.0f;
  c.stab_smem = 0;
  const int mode = t.dec_in_smem;
  if (chunk_path_ok(c, mode, sym_dtype, symbols)) {
    const bool per = g.ib_shift == 0;
    const int r = sym_dtype == RANS_SYM_UINT8
                      ? (per ? launch_decode_chunk<uint8_t, true>(c, st)
                             : launch_decode_chunk<uint8_t, false>(c, st))
                  : sym_dtype == RANS_SYM_INT16
                      ? (per ? launch_decode_chunk<int16_t, true>(c, st)
                             : launch_decode_chunk<int16_t, false>(c, st))
                      : (per ? launch_decode_chunk<int32_t, true>(c, st)
                             : launch_decode_chunk<int32_t, false>(c, st));
    if (r != kNotTaken) return r;
  }
  if (tile_path_ok(c, mode, sym_dtype, indexes, symbols)) {
    const int r = g.fmt == RANS_FMT_RANS32_16 ? launch_decode_tile<Rans32>(c, indexes, symbols, st)
                                              : launch_decode_tile<Rans64>(c, indexes, symbols, st);
    if (r != kNotTaken) return r;
  }
  switch (sym_dtype) {
    case RANS_SYM_INT32: return launch_decode_s<int32_t>(c, mode, st);
    case RANS_SYM_UINT8: return launch_decode_s<uint8_t>(c, mode, st);
    case RANS_SYM_INT16: return launch_decode_s<int16_t>(c, mode, st);
    default: return RANS_ERR_ARG;
  }
}

}  // namespace rb
