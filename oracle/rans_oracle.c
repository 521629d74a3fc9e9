/*
 * rans_oracle.c -- the correctness oracle for indexed 64-bit rANS coding.
 *
 * TEST INFRASTRUCTURE ONLY.  This is a plain, slow, single-threaded CPU
 * restatement of the method, written from the prose of the pages below.  It
 * shares no code, header, table or constant generator with the CUDA library
 * (rans_entropy_coding_b200/csrc).  Only tests/, the smoke check and the
 * bench's CPU-baseline leg may load it; the product path never does.
 *
 * Sources (page title, then section):
 *   [KR]  "kompressor" README (docs.rs crate source) -- Highlights, Why,
 *         Correctness, Credits: 64-bit rANS in the ryg_rans style, a byte-exact
 *         port of CompressAI's coder, bypass path for outliers, independent
 *         chunks.
 *   [KB]  kompressor "Benchmark notes: why the entropy coder, not the
 *         architecture" -- section 4: the decoder looks a symbol up with a
 *         linear scan over the CDF row.
 *   [TA]  "torch_ans 0.3.0" (PyPI) -- Usage (variants table: rans64 has a
 *         64-bit state, 32-bit stream words, 16-bit frequencies), Low-level
 *         API (rans_push / rans_pop: cdfs, cdfs_sizes, offsets, bypass coding,
 *         the coded range [offset, offset + cdf_size - 2) and the zig-zag raw
 *         value), High-level API (init_params turns pmfs into quantised CDFs),
 *         FAQ (cdf rows are increasing positive integers below 2^precision;
 *         interleaved states share one sequentially processed bitstream),
 *         Performance Tuning GPU item 5 (bypass is sequential across lanes).
 *
 * Where the pages are silent the plainest reading is taken; each such reading
 * is marked "Reading:" below.
 *
 * Every function is pinned by tests in tests/test_oracle_*.py against
 * hand-worked streams, closed forms, brute force and invariants.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "rans_oracle.h"

/* ---------------------------------------------------------------- O1 ----
 * Constants.  [TA] Usage, rans64 row: 64-bit state, 32-bit stream words,
 * 16-bit frequency precision.  Reading: the lower state bound L is 2^31, the
 * only value for which one 32-bit word brings a state below L back into
 * [L, 2^32 L); the bypass piece is 4 bits wide ([TA] rans_push takes a
 * bypass_precision; 4 is the reading used here).
 */
#define PREC 16u
#define TOTAL (1u << PREC)          /* M = 2^16: the sum of a CDF row */
#define RANS_L (1ull << 31)         /* lower bound of the state */
#define BYPASS_BITS 4u
#define BYPASS_MAX 15u              /* largest bypass piece */

/* ---------------------------------------------------------------- O2 ----
 * pmf -> quantised CDF row.  [TA] High-level API ("Handles CDF/PMF conversion
 * internally"), FAQ (cdf values are increasing positive integers below
 * 2^freq_precision).  The input holds the n probabilities of one row, the
 * last of which is the tail mass that becomes the escape bucket; the output
 * row has n + 1 entries with cdf[0] = 0 and cdf[n] = 2^16.
 *
 * Reading (the pages give no procedure; this is CompressAI's, as commonly
 * described):
 *   1. each probability is scaled to 2^16 and rounded half away from zero;
 *   2. a running sum gives an unnormalised CDF with total T;
 *   3. every entry is rescaled to floor(2^16 * c / T);
 *   4. scanning buckets in ascending order, a bucket left empty takes one unit
 *      from the bucket whose width is the smallest above 1 (the first such
 *      bucket on ties), by shifting the CDF entries between the two.
 */
int orc_pmf_to_cdf(const float *pmf, int n, int32_t *cdf)
{
    return orc_pmf_to_cdf_prec(pmf, n, (int)PREC, cdf);
}

/* The same at precision p (rows summing to 2^p): [TA] Usage, the variants
 * table gives rans32_16 frequencies of at most 15 bits, and the FAQ bounds
 * the cdf values by 2^freq_precision.  Reading: steps 1-4 above with 2^16
 * replaced by 2^p. */
int orc_pmf_to_cdf_prec(const float *pmf, int n, int prec, int32_t *cdf)
{
    if (n < 1 || prec < 1 || prec > 16) return ORC_ERR_ARG;
    const uint32_t total = 1u << prec;
    uint64_t *c = (uint64_t *)calloc((size_t)n + 1, sizeof(uint64_t));
    if (!c) return ORC_ERR_ARG;

    /* steps 1 and 2 */
    c[0] = 0;
    for (int i = 0; i < n; ++i) {
        float scaled = pmf[i] * (float)total;   /* exact: times a power of 2 */
        double r = round((double)scaled);       /* half away from zero */
        if (!(r >= 0.0) || r > 4294967295.0) { free(c); return ORC_ERR_ARG; }
        c[i + 1] = c[i] + (uint64_t)r;
    }
    uint64_t T = c[n];
    if (T == 0) { free(c); return ORC_ERR_ARG; }

    /* step 3 */
    for (int i = 0; i <= n; ++i)
        c[i] = ((uint64_t)total * c[i]) / T;

    /* step 4 */
    for (int i = 0; i < n; ++i) {
        if (c[i] != c[i + 1]) continue;
        uint64_t best = UINT64_MAX;
        int steal = -1;
        for (int j = 0; j < n; ++j) {
            uint64_t w = c[j + 1] - c[j];
            if (w > 1 && w < best) { best = w; steal = j; }
        }
        if (steal < 0) { free(c); return ORC_ERR_ARG; }
        if (steal < i) {
            for (int j = steal + 1; j <= i; ++j) c[j] -= 1;
        } else {
            for (int j = i + 1; j <= steal; ++j) c[j] += 1;
        }
    }
    for (int i = 0; i <= n; ++i) cdf[i] = (int32_t)c[i];
    free(c);
    return ORC_OK;
}

/* ---------------------------------------------------------------- O3 ----
 * Gaussian rows from a scale table.  [KR] Getting Started ("64 cdf rows" for
 * y) and [KB] section 4 ("cdf.tolist() (200512 elements)" = 64 x 3133).
 * Reading: CompressAI's GaussianConditional construction -- for a tail mass t
 * the multiplier is m = -Phi^-1(t/2); a row of scale s has centre
 * ceil(s * m), pmf entries Phi((0.5-|k|)/s) - Phi((-0.5-|k|)/s) for
 * k = -centre..centre, the tail 2 Phi((-0.5-centre)/s), offset -centre and
 * cdf length 2 centre + 3.  Phi is evaluated in double precision and the pmf
 * is cast to float before quantisation.
 */
static double std_normal_cdf(double z)
{
    return 0.5 * erfc(-z / sqrt(2.0));
}

double orc_gaussian_multiplier(double tail_mass)
{
    /* Phi^-1(t/2) by bisection: Phi is increasing, so halve [lo, hi] until
     * the midpoint no longer moves. */
    double target = tail_mass / 2.0;
    double lo = -40.0, hi = 0.0;
    for (int it = 0; it < 400; ++it) {
        double mid = 0.5 * (lo + hi);
        if (mid == lo || mid == hi) break;
        if (std_normal_cdf(mid) < target) lo = mid; else hi = mid;
    }
    /* the point closer to the root; ties to the upper end */
    double flo = fabs(std_normal_cdf(lo) - target);
    double fhi = fabs(std_normal_cdf(hi) - target);
    double z = (flo < fhi) ? lo : hi;
    return -z;
}

int orc_gaussian_center(float scale, double tail_mass, int32_t *center)
{
    if (!(scale > 0.0f) || !(tail_mass > 0.0) || !(tail_mass < 1.0)) return ORC_ERR_ARG;
    double m = orc_gaussian_multiplier(tail_mass);
    double c = ceil((double)scale * m);
    if (c < 0.0 || c > 32766.0) return ORC_ERR_ARG;
    *center = (int32_t)c;
    return ORC_OK;
}

int orc_build_cdfs_from_scales(const float *scales, int K, double tail_mass,
                               int32_t *cdfs, int Lmax, int32_t *lengths,
                               int32_t *offsets)
{
    return orc_build_cdfs_from_scales_prec(scales, K, tail_mass, (int)PREC, cdfs, Lmax,
                                           lengths, offsets);
}

int orc_build_cdfs_from_scales_prec(const float *scales, int K, double tail_mass, int prec,
                                    int32_t *cdfs, int Lmax, int32_t *lengths,
                                    int32_t *offsets)
{
    if (K <= 0 || Lmax < 3) return ORC_ERR_ARG;
    for (int r = 0; r < K; ++r) {
        int32_t center;
        int st = orc_gaussian_center(scales[r], tail_mass, &center);
        if (st) return st;
        int npmf = 2 * center + 1;
        int len = npmf + 2;
        if (len > Lmax) return ORC_ERR_CAPACITY;
        float *p = (float *)malloc(sizeof(float) * (size_t)(npmf + 1));
        if (!p) return ORC_ERR_ARG;
        double s = (double)scales[r];
        for (int k = 0; k < npmf; ++k) {
            double d = fabs((double)(k - center));
            double upper = std_normal_cdf((0.5 - d) / s);
            double lower = std_normal_cdf((-0.5 - d) / s);
            p[k] = (float)(upper - lower);
        }
        p[npmf] = (float)(2.0 * std_normal_cdf((-0.5 - (double)center) / s));
        int32_t *row = cdfs + (size_t)r * (size_t)Lmax;
        for (int j = 0; j < Lmax; ++j) row[j] = 0;
        st = orc_pmf_to_cdf_prec(p, npmf + 1, prec, row);
        free(p);
        if (st) return st;
        lengths[r] = len;
        offsets[r] = -center;
    }
    return ORC_OK;
}

/* Rows given as pmfs ([TA] High-level API, init_params(freqs, num_freqs,
 * offsets)): row r holds pmf_lengths[r] probabilities followed by the row's
 * tail mass, so its cdf length is pmf_lengths[r] + 2.  Padding is zero. */
int orc_build_cdfs_from_pmfs(const float *pmfs, int K, int stride,
                             const int32_t *pmf_lengths, const float *tail_mass,
                             int32_t *cdfs, int Lmax, int32_t *lengths)
{
    return orc_build_cdfs_from_pmfs_prec(pmfs, K, stride, pmf_lengths, tail_mass, (int)PREC,
                                         cdfs, Lmax, lengths);
}

int orc_build_cdfs_from_pmfs_prec(const float *pmfs, int K, int stride,
                                  const int32_t *pmf_lengths, const float *tail_mass,
                                  int prec, int32_t *cdfs, int Lmax, int32_t *lengths)
{
    if (K <= 0 || stride <= 0) return ORC_ERR_ARG;
    for (int r = 0; r < K; ++r) {
        int n = pmf_lengths[r];
        if (n < 0 || n > stride) return ORC_ERR_ARG;
        if (n + 2 > Lmax) return ORC_ERR_CAPACITY;
        float *p = (float *)malloc(sizeof(float) * (size_t)(n + 1));
        if (!p) return ORC_ERR_ARG;
        memcpy(p, pmfs + (size_t)r * (size_t)stride, sizeof(float) * (size_t)n);
        p[n] = tail_mass[r];
        int32_t *row = cdfs + (size_t)r * (size_t)Lmax;
        for (int j = 0; j < Lmax; ++j) row[j] = 0;
        int st = orc_pmf_to_cdf_prec(p, n + 1, prec, row);
        free(p);
        if (st) return st;
        lengths[r] = n + 2;
    }
    return ORC_OK;
}

/* ---------------------------------------------------------------- O4 ----
 * Symbol -> op list.  [TA] rans_push: a symbol outside the coded range
 * [offset, offset + cdf_size - 2) codes the escape bucket (the row's last
 * bucket, index cdf_size - 2) and then its distance as a zig-zag raw value in
 * bypass pieces; [KR] Correctness ("outlier case that forces the coder's
 * bypass path").  Reading (CompressAI's convention): below the range maps to
 * an odd raw value 2 d - 1, above it to an even one; the raw value is sent as
 * a count of 4-bit pieces (itself in pieces of at most 15, a 15 meaning "more
 * follows") and then the pieces, least significant first; a symbol equal to
 * offset + cdf_size - 2 takes the escape bucket with raw value 0.  Integers
 * are 64-bit, so every int32 input is exact.
 */
typedef struct {
    uint32_t start;   /* SYM: cdf[v] */
    uint32_t freq;    /* SYM: cdf[v+1] - cdf[v]; 0 marks a BITS op */
    uint32_t val;     /* BITS: the 4-bit value */
    int32_t lane;     /* which interleaved state codes it */
    int32_t row;      /* SYM: the row (for the alias mapping) */
} op_t;

typedef struct {
    op_t *ops;
    size_t n, cap;
} oplist_t;

static int push_op(oplist_t *L, op_t o)
{
    if (L->n == L->cap) {
        size_t nc = L->cap ? 2 * L->cap : 1024;
        op_t *p = (op_t *)realloc(L->ops, nc * sizeof(op_t));
        if (!p) return ORC_ERR_ARG;
        L->ops = p;
        L->cap = nc;
    }
    L->ops[L->n++] = o;
    return ORC_OK;
}

static int symbol_ops(int64_t s, int32_t r, int K, const int32_t *cdfs, int Lmax,
                      const int32_t *lengths, const int32_t *offsets, int lane,
                      oplist_t *L)
{
    if (r < 0 || r >= K) return ORC_ERR_INDEX;
    const int32_t *cdf = cdfs + (size_t)r * (size_t)Lmax;
    int64_t Lr = lengths[r];
    int64_t maxv = Lr - 2;
    int64_t v = s - (int64_t)offsets[r];
    uint64_t raw = 0;
    if (v < 0) {
        raw = (uint64_t)(-2 * v - 1);
        v = maxv;
    } else if (v >= maxv) {
        raw = (uint64_t)(2 * (v - maxv));
        v = maxv;
    }
    int64_t freq = (int64_t)cdf[v + 1] - (int64_t)cdf[v];
    if (freq <= 0) return ORC_ERR_ZERO_FREQ;
    op_t o = {(uint32_t)cdf[v], (uint32_t)freq, 0u, lane, r};
    int st = push_op(L, o);
    if (st) return st;
    if (v == maxv) {
        if (raw >> 60) return ORC_ERR_RANGE;
        uint32_t nb = 0;
        while ((raw >> (BYPASS_BITS * nb)) != 0) ++nb;
        uint32_t cnt = nb;
        while (cnt >= BYPASS_MAX) {
            op_t b = {0u, 0u, BYPASS_MAX, lane, r};
            if ((st = push_op(L, b))) return st;
            cnt -= BYPASS_MAX;
        }
        op_t b = {0u, 0u, cnt, lane, r};
        if ((st = push_op(L, b))) return st;
        for (uint32_t j = 0; j < nb; ++j) {
            op_t piece = {0u, 0u, (uint32_t)((raw >> (BYPASS_BITS * j)) & BYPASS_MAX), lane, r};
            if ((st = push_op(L, piece))) return st;
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------- alias ----
 * Alias coding ([TA] Usage, Alias Coding: it changes both push and pop, pop
 * finding the symbol in constant time; Performance Tuning, GPU items 2-4:
 * the bucket count of a row (cdf size - 1) must be a power of two, and push
 * reads a remap table that spans the whole 2^precision range).  Reading
 * (the pages give no construction): the 2^p cumulative positions are cut
 * into n = cdf size - 1 slots of B = 2^p / n positions; slot j holds
 * positions [jB, jB + d_j) of symbol j and the rest of the slot for symbol
 * a_j.  The d_j and a_j come from Vose's alias method on the frequencies f_s:
 * symbols with f < B form the small list and those with f > B the large one,
 * both in ascending order and worked first-in first-out; the head of small
 * keeps d = its remaining frequency and takes the head of large as its alias,
 * which gives up B - d and moves to the back of small once below B (and is
 * done, d = B, at exactly B).  Within symbol s the positions are ranked:
 * first its own slot's [0, d_s), then its alias parts in slot order.
 * Encoding codes symbol s on the position of rank x mod f_s (instead of
 * cdf[s] + x mod f_s); decoding finds the slot of x mod 2^p, its symbol and
 * rank.  A row whose every frequency is B reduces to the plain coder.
 */
typedef struct {
    int logB;        /* log2 of the slot width B */
    int32_t *d;      /* per slot: positions of the slot's own symbol */
    int32_t *a;      /* per slot: the alias symbol of the rest */
    int32_t *base;   /* per slot: rank (within a_j) of the rest's first position */
    int32_t *remap;  /* 2^p entries: remap[cdf[s] + r] = position of rank r of s */
} alias_t;

int orc_alias_build(const int32_t *cdf, int len, int prec, int32_t *d, int32_t *a,
                    int32_t *base, int32_t *remap)
{
    const int n = len - 1;
    if (n < 1 || (n & (n - 1)) != 0 || prec < 1 || prec > 16) return ORC_ERR_ARG;
    const int32_t M = (int32_t)1 << prec;
    if (n > M || cdf[0] != 0 || cdf[n] != M) return ORC_ERR_ARG;
    const int32_t B = M / n;
    int32_t *rem = (int32_t *)malloc(sizeof(int32_t) * (size_t)n);
    int32_t *small = (int32_t *)malloc(sizeof(int32_t) * (size_t)n);
    int32_t *large = (int32_t *)malloc(sizeof(int32_t) * (size_t)n);
    int32_t *cnt = (int32_t *)malloc(sizeof(int32_t) * (size_t)n);
    int st = ORC_OK;
    if (!rem || !small || !large || !cnt) { st = ORC_ERR_ARG; goto done; }
    int ns = 0, nl = 0, hs = 0, hl = 0;
    for (int j = 0; j < n; ++j) {
        const int32_t f = cdf[j + 1] - cdf[j];
        if (f <= 0) { st = ORC_ERR_ZERO_FREQ; goto done; }
        rem[j] = f;
        d[j] = B;
        a[j] = j;
        base[j] = 0;
        if (f < B) small[ns++] = j;
        else if (f > B) large[nl++] = j;
    }
    while (hs < ns && hl < nl) {
        const int32_t l = small[hs++];
        const int32_t g = large[hl];
        d[l] = rem[l];
        a[l] = g;
        rem[g] -= B - rem[l];
        if (rem[g] <= B) {
            ++hl;
            if (rem[g] < B) small[ns++] = g;   /* at exactly B it keeps d = B */
        }
    }
    if (hs < ns || hl < nl) { st = ORC_ERR_ARG; goto done; }   /* cannot happen */
    /* ranks: own part first, then alias parts in slot order */
    for (int j = 0; j < n; ++j) cnt[j] = d[j];
    for (int j = 0; j < n; ++j) {
        if (d[j] == B) continue;
        base[j] = cnt[a[j]];
        cnt[a[j]] += B - d[j];
    }
    for (int j = 0; j < n; ++j)
        if (cnt[j] != cdf[j + 1] - cdf[j]) { st = ORC_ERR_ARG; goto done; }
    if (remap) {
        for (int j = 0; j < n; ++j) {
            for (int32_t o = 0; o < B; ++o) {
                const int32_t pos = j * B + o;
                if (o < d[j]) remap[cdf[j] + o] = pos;
                else remap[cdf[a[j]] + base[j] + (o - d[j])] = pos;
            }
        }
    }
done:
    free(rem);
    free(small);
    free(large);
    free(cnt);
    return st;
}

/* Alias tables of all K rows (NULL on error: a row whose bucket count is not
 * a power of two, or a malformed row). */
static alias_t *alias_tables(const int32_t *cdfs, int K, int Lmax, const int32_t *lengths,
                             int prec)
{
    alias_t *al = (alias_t *)calloc((size_t)K, sizeof(alias_t));
    if (!al) return NULL;
    for (int r = 0; r < K; ++r) {
        const int n = lengths[r] - 1;
        const int32_t M = (int32_t)1 << prec;
        al[r].d = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n > 0 ? n : 1));
        al[r].a = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n > 0 ? n : 1));
        al[r].base = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n > 0 ? n : 1));
        al[r].remap = (int32_t *)malloc(sizeof(int32_t) * (size_t)M);
        int lb = 0;
        while (n > 0 && (M / n) > (1 << lb)) ++lb;
        al[r].logB = lb;
        if (!al[r].d || !al[r].a || !al[r].base || !al[r].remap ||
            orc_alias_build(cdfs + (size_t)r * (size_t)Lmax, lengths[r], prec, al[r].d, al[r].a,
                            al[r].base, al[r].remap) != ORC_OK) {
            for (int q = 0; q <= r; ++q) {
                free(al[q].d); free(al[q].a); free(al[q].base); free(al[q].remap);
            }
            free(al);
            return NULL;
        }
    }
    return al;
}

static void alias_free(alias_t *al, int K)
{
    if (!al) return;
    for (int r = 0; r < K; ++r) {
        free(al[r].d); free(al[r].a); free(al[r].base); free(al[r].remap);
    }
    free(al);
}

/* The position a SYM op codes on: cdf[s] + rank, or the alias position of
 * that rank. */
static uint32_t code_position(const alias_t *al, const op_t *o, uint64_t rank)
{
    return al ? (uint32_t)al[o->row].remap[o->start + rank] : o->start + (uint32_t)rank;
}

/* The alias decoder's symbol and rank of position c in row r. */
static void alias_lookup(const alias_t *al, int r, uint32_t c, int32_t *v, uint32_t *rank)
{
    const alias_t *t = &al[r];
    const uint32_t j = c >> t->logB;
    const uint32_t o = c & ((1u << t->logB) - 1u);
    if (o < (uint32_t)t->d[j]) {
        *v = (int32_t)j;
        *rank = o;
    } else {
        *v = t->a[j];
        *rank = (uint32_t)t->base[j] + (o - (uint32_t)t->d[j]);
    }
}

/* ------------------------------------------------------------ O5 / O7 ----
 * Encode one stream.  [KR] Credits (ryg_rans 64-bit coder), [TA] FAQ
 * (interleaved states share one bitstream that is processed sequentially).
 * The op list of symbols 0..n-1 is coded in reverse order; op k belongs to
 * lane (symbol index mod W).  SYM(start, freq): if x >= 2^47 freq, push the
 * low 32 bits and shift x right by 32; then x = (x / freq) 2^16 + x mod freq
 * + start.  BITS(v): if x >= 2^59, push a word likewise; then x = 16 x + v.
 * Flush: lanes W-1 .. 0 push their state as two words, high first.  The
 * stream is the pushed words in reverse push order, each little-endian.
 * Reading: lane = symbol index mod W and lane 0 first in the flush.  W is 1,
 * 2, 4, 8 ([TA] Usage, variants table: rans64 interleaves 1, 2, 4 or 8
 * states) or 32 (the warp-wide interleave of the same table's rans32_16
 * row, applied to this format).
 */
static int valid_interleave(int W)
{
    return W == 1 || W == 2 || W == 4 || W == 8 || W == 32;
}

typedef struct {
    uint32_t *w;
    size_t n, cap;
} words_t;

static int push_word(words_t *W, uint32_t v)
{
    if (W->n == W->cap) {
        size_t nc = W->cap ? 2 * W->cap : 1024;
        uint32_t *p = (uint32_t *)realloc(W->w, nc * sizeof(uint32_t));
        if (!p) return ORC_ERR_ARG;
        W->w = p;
        W->cap = nc;
    }
    W->w[W->n++] = v;
    return ORC_OK;
}

static int64_t encode64(const int64_t *sym, const int32_t *row, int64_t n,
                        const int32_t *cdfs, int K, int Lmax,
                        const int32_t *lengths, const int32_t *offsets,
                        int W, uint8_t *out, int64_t cap, const alias_t *al)
{
    if (!valid_interleave(W)) return ORC_ERR_ARG;
    if (n < 0) return ORC_ERR_ARG;
    oplist_t ops = {NULL, 0, 0};
    words_t words = {NULL, 0, 0};
    int64_t result = ORC_OK;

    for (int64_t i = 0; i < n; ++i) {
        int st = symbol_ops(sym[i], row[i], K, cdfs, Lmax, lengths, offsets,
                            (int)(i % W), &ops);
        if (st) { result = st; goto done; }
    }

    uint64_t x[32];
    for (int l = 0; l < W; ++l) x[l] = RANS_L;

    for (size_t k = ops.n; k-- > 0;) {
        const op_t *o = &ops.ops[k];
        uint64_t *s = &x[o->lane];
        if (o->freq) {
            uint64_t xmax = ((uint64_t)1 << 47) * (uint64_t)o->freq;
            if (*s >= xmax) {
                if (push_word(&words, (uint32_t)*s)) { result = ORC_ERR_ARG; goto done; }
                *s >>= 32;
            }
            *s = ((*s / o->freq) << PREC) + code_position(al, o, *s % o->freq);
        } else {
            uint64_t xmax = (uint64_t)1 << 59;
            if (*s >= xmax) {
                if (push_word(&words, (uint32_t)*s)) { result = ORC_ERR_ARG; goto done; }
                *s >>= 32;
            }
            *s = (*s << BYPASS_BITS) | o->val;
        }
    }
    for (int l = W - 1; l >= 0; --l) {
        if (push_word(&words, (uint32_t)(x[l] >> 32)) ||
            push_word(&words, (uint32_t)x[l])) { result = ORC_ERR_ARG; goto done; }
    }

    int64_t nbytes = (int64_t)words.n * 4;
    if (nbytes > cap) { result = ORC_ERR_CAPACITY; goto done; }
    for (size_t k = 0; k < words.n; ++k) {
        uint32_t v = words.w[words.n - 1 - k];
        out[4 * k + 0] = (uint8_t)(v);
        out[4 * k + 1] = (uint8_t)(v >> 8);
        out[4 * k + 2] = (uint8_t)(v >> 16);
        out[4 * k + 3] = (uint8_t)(v >> 24);
    }
    result = nbytes;
done:
    free(ops.ops);
    free(words.w);
    return result;
}

/* ------------------------------------------------------------ O6 / O7 ----
 * Decode one stream.  [KB] section 4: the symbol is found by a linear scan
 * of the row -- the first j >= 1 with cdf[j] > cum, minus one.  Then
 * x = freq (x >> 16) + cum - start, and a state below L takes the next word
 * as its low 32 bits.  An escape reads the bypass count and pieces the same
 * way, 4 bits at a time.  Symbols 0..n-1 are decoded in order, each on lane
 * i mod W, refilling from one shared cursor.  The stream must end exactly
 * where its words end with every lane back at L (the encoder's start); any
 * other ending, or a read past the end, is reported as corrupt.
 */
typedef struct {
    const uint8_t *p;
    int64_t len, pos;
} reader_t;

static int read_word(reader_t *R, uint32_t *v)
{
    if (R->pos + 4 > R->len) return ORC_ERR_CORRUPT;
    const uint8_t *b = R->p + R->pos;
    *v = (uint32_t)b[0] | ((uint32_t)b[1] << 8) | ((uint32_t)b[2] << 16) |
         ((uint32_t)b[3] << 24);
    R->pos += 4;
    return ORC_OK;
}

static int refill(uint64_t *x, reader_t *R)
{
    if (*x < RANS_L) {
        uint32_t w;
        int st = read_word(R, &w);
        if (st) return st;
        *x = (*x << 32) | w;
    }
    return ORC_OK;
}

static int get_bits(uint64_t *x, reader_t *R, uint32_t *val)
{
    *val = (uint32_t)(*x & BYPASS_MAX);
    *x >>= BYPASS_BITS;
    return refill(x, R);
}

static int decode64(const uint8_t *in, int64_t len, const int32_t *row, int64_t n,
                    const int32_t *cdfs, int K, int Lmax,
                    const int32_t *lengths, const int32_t *offsets,
                    int W, int64_t *sym_out, const alias_t *al)
{
    if (!valid_interleave(W)) return ORC_ERR_ARG;
    reader_t R = {in, len, 0};
    uint64_t x[32];
    for (int l = 0; l < W; ++l) {
        uint32_t lo, hi;
        if (read_word(&R, &lo) || read_word(&R, &hi)) return ORC_ERR_CORRUPT;
        x[l] = ((uint64_t)hi << 32) | lo;
    }
    for (int64_t i = 0; i < n; ++i) {
        int32_t r = row[i];
        if (r < 0 || r >= K) return ORC_ERR_INDEX;
        const int32_t *cdf = cdfs + (size_t)r * (size_t)Lmax;
        int32_t Lr = lengths[r];
        int32_t maxv = Lr - 2;
        uint64_t *s = &x[i % W];

        uint32_t cum = (uint32_t)(*s & (TOTAL - 1));
        int32_t v;
        uint32_t rank;
        if (al) {
            alias_lookup(al, r, cum, &v, &rank);
        } else {
            int j = 1;
            while (j < Lr && (uint32_t)cdf[j] <= cum) ++j;
            if (j >= Lr) return ORC_ERR_CORRUPT;    /* a malformed row */
            v = j - 1;
            rank = cum - (uint32_t)cdf[v];
        }
        uint32_t freq = (uint32_t)(cdf[v + 1] - cdf[v]);
        *s = (uint64_t)freq * (*s >> PREC) + rank;
        int st = refill(s, &R);
        if (st) return st;

        int64_t value = v;
        if (v == maxv) {
            uint32_t val;
            if ((st = get_bits(s, &R, &val))) return st;
            uint32_t nb = val;
            while (val == BYPASS_MAX) {
                if ((st = get_bits(s, &R, &val))) return st;
                nb += val;
            }
            if (nb > 15) return ORC_ERR_CORRUPT;   /* raw would exceed 60 bits */
            uint64_t raw = 0;
            for (uint32_t k = 0; k < nb; ++k) {
                if ((st = get_bits(s, &R, &val))) return st;
                raw |= (uint64_t)val << (BYPASS_BITS * k);
            }
            int64_t half = (int64_t)(raw >> 1);
            value = (raw & 1) ? (-half - 1) : ((int64_t)maxv + half);
        }
        sym_out[i] = value + (int64_t)offsets[r];
    }
    if (R.pos != R.len) return ORC_ERR_CORRUPT;
    for (int l = 0; l < W; ++l)
        if (x[l] != RANS_L) return ORC_ERR_CORRUPT;
    return ORC_OK;
}

int64_t orc_encode_stream(const int64_t *sym, const int32_t *row, int64_t n,
                          const int32_t *cdfs, int K, int Lmax,
                          const int32_t *lengths, const int32_t *offsets,
                          int W, uint8_t *out, int64_t cap)
{
    return encode64(sym, row, n, cdfs, K, Lmax, lengths, offsets, W, out, cap, NULL);
}

int orc_decode_stream(const uint8_t *in, int64_t len, const int32_t *row, int64_t n,
                      const int32_t *cdfs, int K, int Lmax,
                      const int32_t *lengths, const int32_t *offsets,
                      int W, int64_t *sym_out)
{
    return decode64(in, len, row, n, cdfs, K, Lmax, lengths, offsets, W, sym_out, NULL);
}

/* ------------------------------------------------------------ rans32_16 ----
 * The 32-bit-state variant.  [TA] Usage, variants table: rans32_16 keeps a
 * 32-bit state, emits 16-bit stream words and takes frequencies of at most 15
 * bits (state bits > stream bits + frequency bits); its interleaved forms use
 * 1, 2, 4, 8 or 32 states per stream, one shared stream of words ([TA] FAQ).
 * Reading, by the same argument as O1: the lower bound is L16 = 2^16, the
 * only value for which one 16-bit word brings a state below it back into
 * [L16, 2^16 L16).  So, with rows summing to 2^p (1 <= p <= 15):
 *   SYM(start, freq): if x >= 2^(32-p) freq, push the low 16 bits and shift x
 *     right by 16; then x = (x / freq) 2^p + x mod freq + start;
 *   BITS(v): if x >= 2^28, push a word likewise; then x = 16 x + v;
 *   flush: lanes W-1 .. 0 push their state as two 16-bit words, high first;
 *   the stream is the words in reverse push order, each little-endian, so it
 *   starts with lane 0's low and high halves.  The symbol -> op mapping (O4)
 *   and the lane of a symbol (index mod W) are those of the 64-bit coder.
 * Decoding mirrors it: cum = x mod 2^p, the linear scan of [KB] section 4,
 * x = freq (x >> p) + cum - start, and a state below 2^16 takes the next word
 * as its low 16 bits.
 */
#define R16_L (1u << 16)

typedef struct {
    uint16_t *w;
    size_t n, cap;
} words16_t;

static int push_word16(words16_t *W, uint16_t v)
{
    if (W->n == W->cap) {
        size_t nc = W->cap ? 2 * W->cap : 1024;
        uint16_t *p = (uint16_t *)realloc(W->w, nc * sizeof(uint16_t));
        if (!p) return ORC_ERR_ARG;
        W->w = p;
        W->cap = nc;
    }
    W->w[W->n++] = v;
    return ORC_OK;
}


static int64_t encode16(const int64_t *sym, const int32_t *row, int64_t n,
                        const int32_t *cdfs, int K, int Lmax,
                        const int32_t *lengths, const int32_t *offsets,
                        int prec, int W, uint8_t *out, int64_t cap, const alias_t *al)
{
    if (!valid_interleave(W) || n < 0 || prec < 1 || prec > 15) return ORC_ERR_ARG;
    oplist_t ops = {NULL, 0, 0};
    words16_t words = {NULL, 0, 0};
    int64_t result = ORC_OK;

    for (int64_t i = 0; i < n; ++i) {
        int st = symbol_ops(sym[i], row[i], K, cdfs, Lmax, lengths, offsets,
                            (int)(i % W), &ops);
        if (st) { result = st; goto done; }
    }

    uint32_t x[32];
    for (int l = 0; l < W; ++l) x[l] = R16_L;

    for (size_t k = ops.n; k-- > 0;) {
        const op_t *o = &ops.ops[k];
        uint32_t *s = &x[o->lane];
        uint64_t xmax = o->freq ? ((uint64_t)o->freq << (32 - prec)) : ((uint64_t)1 << 28);
        if ((uint64_t)*s >= xmax) {
            if (push_word16(&words, (uint16_t)*s)) { result = ORC_ERR_ARG; goto done; }
            *s >>= 16;
        }
        if (o->freq)
            *s = ((*s / o->freq) << prec) + code_position(al, o, *s % o->freq);
        else
            *s = (*s << BYPASS_BITS) | o->val;
    }
    for (int l = W - 1; l >= 0; --l) {
        if (push_word16(&words, (uint16_t)(x[l] >> 16)) ||
            push_word16(&words, (uint16_t)x[l])) { result = ORC_ERR_ARG; goto done; }
    }

    int64_t nbytes = (int64_t)words.n * 2;
    if (nbytes > cap) { result = ORC_ERR_CAPACITY; goto done; }
    for (size_t k = 0; k < words.n; ++k) {
        uint16_t v = words.w[words.n - 1 - k];
        out[2 * k + 0] = (uint8_t)(v);
        out[2 * k + 1] = (uint8_t)(v >> 8);
    }
    result = nbytes;
done:
    free(ops.ops);
    free(words.w);
    return result;
}

static int read_word16(reader_t *R, uint32_t *v)
{
    if (R->pos + 2 > R->len) return ORC_ERR_CORRUPT;
    const uint8_t *b = R->p + R->pos;
    *v = (uint32_t)b[0] | ((uint32_t)b[1] << 8);
    R->pos += 2;
    return ORC_OK;
}

static int refill16(uint32_t *x, reader_t *R)
{
    if (*x < R16_L) {
        uint32_t w;
        int st = read_word16(R, &w);
        if (st) return st;
        *x = (*x << 16) | w;
    }
    return ORC_OK;
}

static int get_bits16(uint32_t *x, reader_t *R, uint32_t *val)
{
    *val = *x & BYPASS_MAX;
    *x >>= BYPASS_BITS;
    return refill16(x, R);
}

static int decode16(const uint8_t *in, int64_t len, const int32_t *row, int64_t n,
                    const int32_t *cdfs, int K, int Lmax,
                    const int32_t *lengths, const int32_t *offsets,
                    int prec, int W, int64_t *sym_out, const alias_t *al)
{
    if (!valid_interleave(W) || prec < 1 || prec > 15) return ORC_ERR_ARG;
    reader_t R = {in, len, 0};
    uint32_t x[32];
    for (int l = 0; l < W; ++l) {
        uint32_t lo, hi;
        if (read_word16(&R, &lo) || read_word16(&R, &hi)) return ORC_ERR_CORRUPT;
        x[l] = (hi << 16) | lo;
    }
    const uint32_t mask = (1u << prec) - 1u;
    for (int64_t i = 0; i < n; ++i) {
        int32_t r = row[i];
        if (r < 0 || r >= K) return ORC_ERR_INDEX;
        const int32_t *cdf = cdfs + (size_t)r * (size_t)Lmax;
        int32_t Lr = lengths[r];
        int32_t maxv = Lr - 2;
        uint32_t *s = &x[i % W];

        uint32_t cum = *s & mask;
        int32_t v;
        uint32_t rank;
        if (al) {
            alias_lookup(al, r, cum, &v, &rank);
        } else {
            int j = 1;
            while (j < Lr && (uint32_t)cdf[j] <= cum) ++j;
            if (j >= Lr) return ORC_ERR_CORRUPT;    /* a malformed row */
            v = j - 1;
            rank = cum - (uint32_t)cdf[v];
        }
        uint32_t freq = (uint32_t)(cdf[v + 1] - cdf[v]);
        *s = freq * (*s >> prec) + rank;
        int st = refill16(s, &R);
        if (st) return st;

        int64_t value = v;
        if (v == maxv) {
            uint32_t val;
            if ((st = get_bits16(s, &R, &val))) return st;
            uint32_t nb = val;
            while (val == BYPASS_MAX) {
                if ((st = get_bits16(s, &R, &val))) return st;
                nb += val;
            }
            if (nb > 15) return ORC_ERR_CORRUPT;   /* raw would exceed 60 bits */
            uint64_t raw = 0;
            for (uint32_t k = 0; k < nb; ++k) {
                if ((st = get_bits16(s, &R, &val))) return st;
                raw |= (uint64_t)val << (BYPASS_BITS * k);
            }
            int64_t half = (int64_t)(raw >> 1);
            value = (raw & 1) ? (-half - 1) : ((int64_t)maxv + half);
        }
        sym_out[i] = value + (int64_t)offsets[r];
    }
    if (R.pos != R.len) return ORC_ERR_CORRUPT;
    for (int l = 0; l < W; ++l)
        if (x[l] != R16_L) return ORC_ERR_CORRUPT;
    return ORC_OK;
}

int64_t orc_encode_stream16(const int64_t *sym, const int32_t *row, int64_t n,
                            const int32_t *cdfs, int K, int Lmax,
                            const int32_t *lengths, const int32_t *offsets,
                            int prec, int W, uint8_t *out, int64_t cap)
{
    return encode16(sym, row, n, cdfs, K, Lmax, lengths, offsets, prec, W, out, cap, NULL);
}

int orc_decode_stream16(const uint8_t *in, int64_t len, const int32_t *row, int64_t n,
                        const int32_t *cdfs, int K, int Lmax,
                        const int32_t *lengths, const int32_t *offsets,
                        int prec, int W, int64_t *sym_out)
{
    return decode16(in, len, row, n, cdfs, K, Lmax, lengths, offsets, prec, W, sym_out, NULL);
}

/* Alias-coded streams (see "alias" above) in either format: prec 16 codes
 * the 64-bit format, prec <= 15 the rans32_16 one.  Every row's bucket count
 * must be a power of two (else ORC_ERR_ARG).  The pages list the alias coder
 * for 1, 2, 4 and 8 interleaved states. */
int64_t orc_encode_stream_alias(const int64_t *sym, const int32_t *row, int64_t n,
                                const int32_t *cdfs, int K, int Lmax,
                                const int32_t *lengths, const int32_t *offsets,
                                int prec, int W, uint8_t *out, int64_t cap)
{
    if (W != 1 && W != 2 && W != 4 && W != 8) return ORC_ERR_ARG;
    alias_t *al = alias_tables(cdfs, K, Lmax, lengths, prec);
    if (!al) return ORC_ERR_ARG;
    int64_t st = prec == 16
        ? encode64(sym, row, n, cdfs, K, Lmax, lengths, offsets, W, out, cap, al)
        : encode16(sym, row, n, cdfs, K, Lmax, lengths, offsets, prec, W, out, cap, al);
    alias_free(al, K);
    return st;
}

int orc_decode_stream_alias(const uint8_t *in, int64_t len, const int32_t *row, int64_t n,
                            const int32_t *cdfs, int K, int Lmax,
                            const int32_t *lengths, const int32_t *offsets,
                            int prec, int W, int64_t *sym_out)
{
    if (W != 1 && W != 2 && W != 4 && W != 8) return ORC_ERR_ARG;
    alias_t *al = alias_tables(cdfs, K, Lmax, lengths, prec);
    if (!al) return ORC_ERR_ARG;
    int st = prec == 16
        ? decode64(in, len, row, n, cdfs, K, Lmax, lengths, offsets, W, sym_out, al)
        : decode16(in, len, row, n, cdfs, K, Lmax, lengths, offsets, prec, W, sym_out, al);
    alias_free(al, K);
    return st;
}
