// tables.cu -- CDF-table construction and the coder's prepared tables.
//
//  * Gaussian rows from a scale table ("kompressor" README, Getting Started:
//    64 CDF rows for the y latent; "Benchmark notes", section 4: 200512 table
//    entries = 64 rows x 3133).
//  * pmf -> quantised CDF ("torch_ans 0.3.0", High-level API, init_params;
//    FAQ: increasing positive integers up to 2^precision).
//  * The decoder lookup table: the top q bits of the state's low 16 bits pick
//    a slot that resolves up to two bucket boundaries itself and points to
//    boundary bitmaps when it holds more ("torch_ans 0.3.0", Usage:
//    inverse-CDF decoding with a 2^q table instead of a search).
//
// One CUDA block quantises one row.  The steal step (every empty bucket takes
// one unit from the narrowest bucket wider than 1, first on ties, in ascending
// order of empty buckets) is computed in closed form: the units come from the
// buckets in (width, index) order, each drained to width 1 before the next is
// touched, so a threshold width t and a rank among the width-t buckets decide
// every bucket's final width.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <vector>

#include "rans_common.cuh"
#include "rans_internal.h"

namespace rb {

namespace {

constexpr int kRowThreads = 1024;
static_assert(kRowThreads == 1024, "one lane per warp total in the block scan");

// Block-wide exclusive scan of a 64-bit value over kRowThreads threads (warp
// shuffles, then every warp scans the 32 warp totals); *total gets the block
// sum.
struct BlockScratch {
  unsigned long long warp[kRowThreads / 32];
  unsigned long long total;
  unsigned long long aux;
};

__device__ unsigned long long block_excl_scan(unsigned long long v, BlockScratch &sh,
                                              unsigned long long *total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  unsigned long long inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long t = __shfl_up_sync(kFull, inc, o);
    if (lane >= o) inc += t;
  }
  if (lane == 31) sh.warp[wid] = inc;
  __syncthreads();
  // every warp scans the 32 warp totals itself and takes its own prefix
  const unsigned long long w = sh.warp[lane];
  unsigned long long wi = w;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long t = __shfl_up_sync(kFull, wi, o);
    if (lane >= o) wi += t;
  }
  *total = __shfl_sync(kFull, wi, 31);
  const unsigned long long ex = __shfl_sync(kFull, wi - w, wid) + inc - v;
  __syncthreads();  // every thread has read the scratch before anyone reuses it
  return ex;
}

// Scaled and rounded probability: round(p * total) half away from zero
// (total = 2^precision), or -1 when p is negative, not finite or too large.
__device__ __forceinline__ long long scaled_freq(float p, uint32_t total) {
  float v = p * (float)total;             // exact: times a power of two
  float r = roundf(v);                    // half away from zero
  if (!(r >= 0.0f) || (double)r > 4294967295.0) return -1;
  return (long long)r;
}

// Quantises n probabilities (the last one the tail mass) into row[0..n] of a
// CDF row.  Returns RANS_OK or RANS_ERR_TABLE (same value on every thread).
// Thread t owns the contiguous entries [t * per, (t + 1) * per): each pass
// walks its own entries in order and block scans join the threads.  row[1..n]
// holds first the rounded probabilities (written by pf.eval), then the bucket
// widths, then the CDF.
//
// The steal step in closed form: the Z units that the empty buckets take
// come from the buckets in (width, index) order, each drained to width 1
// before the next is touched.  So with S(t) = sum over buckets of width
// 1 < w <= t of (w - 1), the threshold t is the smallest width with
// S(t) >= Z: buckets narrower than t end at width 1, and of the width-t
// buckets (in index order) the first floor(R / (t - 1)) end at 1 and the
// next gives up R mod (t - 1) units, R = Z - S(t - 1).  Widths below kBins
// are counted in a histogram (one bin per thread, so one scan finds t); the
// wider ones, at most 2^16 / kBins of them, are kept in a list.
constexpr int kBins = kRowThreads;
constexpr int kBigMax = 65536 / kBins;

struct QuantScratch {
  unsigned int hist[kBins];
  unsigned int big[kBigMax];
  unsigned int nbig;
};

// floor(a / T) for T >= 1 and a / T < 2^32 (a = total * c with c <= T):
// the double product a * (1 / T) is within one of the quotient (its
// relative error is a few units of 2^-53 and the quotient is below 2^32),
// and one exact integer step corrects it.
__device__ __forceinline__ unsigned long long div_floor(unsigned long long a,
                                                        unsigned long long T, double rT) {
  unsigned long long q = (unsigned long long)((double)a * rT);
  const long long r = (long long)(a - q * T);
  if (r < 0) --q;
  else if ((unsigned long long)r >= T) ++q;
  return q;
}

template <class PF>
__device__ int quantise_row(const PF &pf, int n, int32_t *row, BlockScratch &sh,
                            QuantScratch &q, uint32_t total) {
  const int per = (n + kRowThreads - 1) / kRowThreads;
  const int i0 = min(n, (int)threadIdx.x * per), i1 = min(n, i0 + per);
  // pass 1: rounded values, each probability evaluated once
  int bad = 0;
  const unsigned long long local = pf.eval(i0, i1, row + 1, bad);
  q.hist[threadIdx.x] = 0;
  if (threadIdx.x == 0) {
    q.nbig = 0;
    sh.total = 0;  // (no threshold found yet; nothing else writes it before)
  }
  // a thread with a bad value adds 2^52 to the total: the rounded values are
  // below 2^32 and at most 2^16 of them, so a good total stays below 2^48,
  // and 1024 flags add up below 2^63
  unsigned long long T;
  const unsigned long long before =
      block_excl_scan(local + (bad ? 1ull << 52 : 0ull), sh, &T);
  if (T == 0 || (T >> 52) != 0) return RANS_ERR_TABLE;

  // pass 2: widths of the rescaled running sum floor(total c / T); count the
  // empty buckets and the widths of the others
  unsigned long long zl = 0;
  {
    const double rT = 1.0 / (double)T;
    unsigned long long c = before;
    unsigned long long b0 = div_floor((unsigned long long)total * c, T, rT);
    for (int i = i0; i < i1; ++i) {
      c += (uint32_t)row[i + 1];
      const unsigned long long b1 = div_floor((unsigned long long)total * c, T, rT);
      const uint32_t w = (uint32_t)(b1 - b0);
      b0 = b1;
      row[i + 1] = (int32_t)w;
      zl += (w == 0);
      if (w >= 2 && w < (uint32_t)kBins) atomicAdd(&q.hist[w], 1u);
      else if (w >= (uint32_t)kBins) q.big[atomicAdd(&q.nbig, 1u)] = w;
    }
  }
  __syncthreads();  // every thread's bins and wide buckets are in
  // one scan gives Z (the empty buckets, high half) and, over the bins
  // (thread b = width b), S(b - 1) and S(kBins - 1) (low half): both sums
  // stay below 2^32
  const unsigned int b = threadIdx.x;
  const unsigned long long vb = b >= 2 ? (unsigned long long)(b - 1) * q.hist[b] : 0ull;
  unsigned long long zs;
  const unsigned long long exz = block_excl_scan((zl << 32) | vb, sh, &zs);
  const unsigned long long Z = zs >> 32;
  if (Z > 0) {
    // t below kBins: the bin whose running S(t) first reaches Z
    const unsigned long long sb = exz & 0xffffffffull;     // S(b - 1)
    const unsigned long long s_all = zs & 0xffffffffull;   // S(kBins - 1)
    if (vb > 0 && sb < Z && sb + vb >= Z) {
      sh.total = b;
      sh.aux = sb;
    }
    // t among the wide buckets: the smallest listed width whose S reaches Z
    const unsigned int nbig = q.nbig;
    if (s_all < Z && b < nbig) {
      const unsigned int wb = q.big[b];
      unsigned long long s_le = s_all, s_lt = s_all;  // S(wb), S(wb - 1)
      for (unsigned int k = 0; k < nbig; ++k) {
        const unsigned int wk = q.big[k];
        if (wk <= wb) s_le += wk - 1;
        if (wk < wb) s_lt += wk - 1;
      }
      if (s_le >= Z && s_lt < Z) {  // every bucket of the smallest such width agrees
        sh.total = wb;
        sh.aux = s_lt;
      }
    }
    __syncthreads();
    const long long t = (long long)sh.total;  // (not written again: no barrier after)
    const unsigned long long below = sh.aux;
    if (t == 0) return RANS_ERR_TABLE;  // nothing left to steal from
    const unsigned long long R = Z - below;
    const unsigned long long full = R / (unsigned long long)(t - 1);
    const unsigned long long part = R % (unsigned long long)(t - 1);
    // the final widths and the CDF in one scan: each thread counts its
    // width-t buckets (nt) and adds up its other buckets' final widths (a:
    // 1 below t, their own above); the width-t buckets before it (rank r <
    // rk0, in index order) end at 1 below rank `full`, t - part at it and t
    // above, which sums to g(rk0) in closed form.  (Both counts stay below
    // 2^32, so one 64-bit scan carries them as two halves.)
    unsigned long long nt = 0, a = 0;
    for (int i = i0; i < i1; ++i) {
      const long long w = row[i + 1];
      nt += w == t;
      a += w == t ? 0ull : (w < t ? 1ull : (unsigned long long)w);
    }
    unsigned long long tot;
    const unsigned long long ex = block_excl_scan((a << 32) | nt, sh, &tot);
    unsigned long long rk = ex & 0xffffffffull;
    const unsigned long long g =
        (rk < full ? rk : full) +
        (rk > full ? (unsigned long long)t - part + (rk - full - 1) * (unsigned long long)t : 0ull);
    unsigned long long run = (ex >> 32) + g;
    for (int i = i0; i < i1; ++i) {
      long long w = row[i + 1];
      if (w == t) {
        if (rk < full) w = 1;
        else if (rk == full) w -= (long long)part;
        ++rk;
      } else if (w < t) {
        w = 1;
      }
      run += (unsigned long long)w;
      row[i + 1] = (int32_t)run;
    }
  } else {
    // widths -> CDF in place
    unsigned long long wl = 0;
    for (int i = i0; i < i1; ++i) wl += (uint32_t)row[i + 1];
    unsigned long long tot;
    unsigned long long run = block_excl_scan(wl, sh, &tot);
    for (int i = i0; i < i1; ++i) {
      run += (uint32_t)row[i + 1];
      row[i + 1] = (int32_t)run;
    }
  }
  if (threadIdx.x == 0) row[0] = 0;
  __syncthreads();
  return RANS_OK;
}

// Standard normal CDF as 0.5 erfc(-z / sqrt 2), in double.
__device__ __forceinline__ double std_normal_cdf(double z) {
  return 0.5 * erfc(-z / sqrt(2.0));
}

// The centre ceil(scale m) of a Gaussian row, m = -Phi^-1(tail / 2) (m given:
// gaussian_multiplier(tail)).
__device__ __forceinline__ double gaussian_multiplier(double tail) {
  return -normcdfinv(tail / 2.0);
}

__device__ __forceinline__ int gaussian_center_m(float scale, double tail, double m,
                                                 int32_t *center) {
  if (!(scale > 0.0f) || !isfinite(scale) || !(tail > 0.0) || !(tail < 1.0))
    return RANS_ERR_ARG;
  double c = ceil((double)scale * m);
  if (!(c >= 0.0) || c > 32766.0) return RANS_ERR_ARG;
  *center = (int32_t)c;
  return RANS_OK;
}

__device__ __forceinline__ int gaussian_center(float scale, double tail, int32_t *center) {
  return gaussian_center_m(scale, tail, gaussian_multiplier(tail), center);
}

__global__ void gaussian_lengths_kernel(const float *scales, int K, double tail,
                                        int32_t *lengths, int32_t *offsets) {
  int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= K) return;
  int32_t c = 0;
  int st = gaussian_center(scales[r], tail, &c);
  lengths[r] = st ? st : 2 * c + 3;
  offsets[r] = st ? 0 : -c;
}

// Entry i < npmf of a Gaussian row is Phi((0.5 - d)/s) - Phi((-0.5 - d)/s)
// with d = |i - center|, and entry npmf the tail mass 2 Phi((-0.5 - center)/s).
// With u(d) = Phi((0.5 - d)/s) the entry is u(d) - u(d + 1) (the arguments
// (-0.5 - d) and (0.5 - (d + 1)) are the same double), so a walk over
// consecutive entries evaluates one new u per entry.
struct GaussPmf {
  int center, npmf;
  double s;
  uint32_t total;  // 2^precision
  const double *U;  // u(0 .. center + 1) in shared memory, or null
  __device__ unsigned long long eval(int i0, int i1, int32_t *f, int &bad) const {
    unsigned long long sum = 0;
    if (U) {
      // the row is symmetric about its centre: entry i takes u(d) - u(d + 1),
      // d = |i - centre|, and the tail 2 u(centre + 1) (the same double
      // argument as 2 Phi((-0.5 - centre) / s))
      for (int i = i0; i < i1; ++i) {
        const int d = abs(i - center);
        const float p = i == npmf ? (float)(2.0 * U[center + 1]) : (float)(U[d] - U[d + 1]);
        long long q = scaled_freq(p, total);
        if (q < 0) {
          bad = 1;
          q = 0;
        }
        f[i] = (int32_t)(uint32_t)q;
        sum += (unsigned long long)q;
      }
      return sum;
    }
    int da = -1, db = -1;  // the two most recent u values
    double ua = 0.0, ub = 0.0;
    auto u = [&](int d) -> double {
      if (d == da) return ua;
      if (d == db) return ub;
      const double v = std_normal_cdf((0.5 - (double)d) / s);
      db = da;
      ub = ua;
      da = d;
      ua = v;
      return v;
    };
    for (int i = i0; i < i1; ++i) {
      float p;
      if (i == npmf) {
        p = (float)(2.0 * std_normal_cdf((-0.5 - (double)center) / s));
      } else {
        const int d = abs(i - center);
        const double hi = u(d);
        const double lo = u(d + 1);
        p = (float)(hi - lo);
      }
      long long q = scaled_freq(p, total);
      if (q < 0) {
        bad = 1;
        q = 0;
      }
      f[i] = (int32_t)(uint32_t)q;
      sum += (unsigned long long)q;
    }
    return sum;
  }
};

struct GivenPmf {
  const float *p;
  int n;
  float tail;
  uint32_t total;  // 2^precision
  __device__ unsigned long long eval(int i0, int i1, int32_t *f, int &bad) const {
    unsigned long long sum = 0;
    for (int i = i0; i < i1; ++i) {
      long long q = scaled_freq(i == n ? tail : p[i], total);
      if (q < 0) {
        bad = 1;
        q = 0;
      }
      f[i] = (int32_t)(uint32_t)q;
      sum += (unsigned long long)q;
    }
    return sum;
  }
};

// u(d) = Phi((0.5 - d) / s) for d = 0 .. c + 1 into U (shared memory, c + 2
// doubles), spread over the block; null when they do not fit in cap doubles
// (the row's threads then evaluate their own).
__device__ __forceinline__ const double *gauss_u_table(double *U, int cap, int c, double s) {
  if (c + 2 > cap) return nullptr;  // (uniform)
  for (int d = threadIdx.x; d <= c + 1; d += blockDim.x)
    U[d] = std_normal_cdf((0.5 - (double)d) / s);
  __syncthreads();
  return U;
}

// Dynamic shared memory of the row kernels: the u table (kUTabBytes, Gaussian
// rows only), then the row being quantised (kRowBufEntries entries; longer
// rows are quantised in place in global memory).
constexpr uint32_t kUTabBytes = 32768;
constexpr int kRowBufEntries = 8192;
constexpr uint32_t kRowBufBytes = 4u * kRowBufEntries;
constexpr uint32_t kGaussSmemBytes = kUTabBytes + kRowBufBytes;
static_assert((2u << kMaxQ) <= kUTabBytes, "a row's slot buckets (16-bit) fit in the u table");

// Copies a row quantised in shared memory out to its global row.
__device__ __forceinline__ void write_row(int32_t *row, const int32_t *work, int len) {
  for (int j = threadIdx.x; j < len; j += blockDim.x) row[j] = work[j];
}

__global__ void __launch_bounds__(kRowThreads)
    gaussian_rows_kernel(const float *scales, double tail, int prec, int32_t *cdfs, int Lmax,
                         int32_t *lengths, int32_t *offsets) {
  extern __shared__ __align__(16) double utab[];
  __shared__ BlockScratch sh;
  __shared__ QuantScratch qs;
  int32_t *rbuf = reinterpret_cast<int32_t *>(utab + kUTabBytes / 8);
  const int r = blockIdx.x;
  int32_t *row = cdfs + (size_t)r * (size_t)Lmax;
  int32_t c = 0;
  int st = gaussian_center(scales[r], tail, &c);
  int len = 2 * c + 3;
  if (st == RANS_OK && len > Lmax) st = RANS_ERR_CAPACITY;
  if (st == RANS_OK) {
    const double sd = (double)scales[r];
    const double *U = gauss_u_table(utab, (int)(kUTabBytes / 8), c, sd);
    GaussPmf pf{c, 2 * c + 1, sd, 1u << prec, U};
    int32_t *work = len <= kRowBufEntries ? rbuf : row;
    st = quantise_row(pf, 2 * c + 2, work, sh, qs, 1u << prec);
    if (st == RANS_OK && work != row) write_row(row, work, len);
  }
  for (int j = (st == RANS_OK ? len : 0) + threadIdx.x; j < Lmax; j += kRowThreads) row[j] = 0;
  if (threadIdx.x == 0) {
    lengths[r] = st ? st : len;
    offsets[r] = st ? 0 : -c;
  }
}

__global__ void __launch_bounds__(kRowThreads)
    pmf_rows_kernel(const float *pmfs, int stride, const int32_t *pmf_lengths,
                    const float *tail, int prec, int32_t *cdfs, int Lmax, int32_t *lengths) {
  extern __shared__ __align__(16) int32_t rbuf[];
  __shared__ BlockScratch sh;
  __shared__ QuantScratch qs;
  const int r = blockIdx.x;
  int32_t *row = cdfs + (size_t)r * (size_t)Lmax;
  int n = pmf_lengths[r];
  int st = RANS_OK;
  if (n < 0 || n > stride) st = RANS_ERR_ARG;
  else if (n + 2 > Lmax) st = RANS_ERR_CAPACITY;
  if (st == RANS_OK) {
    GivenPmf pf{pmfs + (size_t)r * (size_t)stride, n, tail[r], 1u << prec};
    int32_t *work = n + 2 <= kRowBufEntries ? rbuf : row;
    st = quantise_row(pf, n + 1, work, sh, qs, 1u << prec);
    if (st == RANS_OK && work != row) write_row(row, work, n + 2);
  }
  for (int j = (st == RANS_OK ? n + 2 : 0) + threadIdx.x; j < Lmax; j += kRowThreads) row[j] = 0;
  if (threadIdx.x == 0) lengths[r] = st ? st : n + 2;
}

// ---- prepared tables ----------------------------------------------------

// Rows of precision p are stored scaled to 16 bits: entry << sh, sh = 16 - p.
// The bucket word of entries a < b: start | (width - 1) << 16, scaled.
__device__ __forceinline__ uint32_t bucket_word(int32_t a, int32_t b, uint32_t sh) {
  return (uint32_t)((a << sh) & 0xffff) | ((uint32_t)(((b - a) << sh) - 1) << 16);
}

// Validates row r and writes its packed buckets.  One block per row.
__global__ void pack_buckets_kernel(const int32_t *cdfs, int Lmax, const RowMeta *meta,
                                    const int32_t *lengths, uint32_t sh, uint32_t *buckets,
                                    uint16_t *starts, int32_t *status) {
  const int r = blockIdx.x;
  const int32_t *row = cdfs + (size_t)r * (size_t)Lmax;
  const int len = lengths[r];
  const int32_t top = (int32_t)(kTotal >> sh);
  const uint32_t base = meta[r * kMetaCopies].bucket_base;
  if (threadIdx.x == 0 && (row[0] != 0 || row[len - 1] != top))
    report(status, RANS_ERR_TABLE, r);
  for (int j = threadIdx.x; j < len - 1; j += blockDim.x) {
    int32_t a = row[j], b = row[j + 1];
    if (!(b > a) || a < 0 || b > top) {
      report(status, RANS_ERR_TABLE, r);
      continue;
    }
    buckets[base + j] = bucket_word(a, b, sh);
  }
  // 16-bit starts, row end included: it writes 0 over the next row's leading
  // 0 (or the trailing sentinel), so overlapping rows agree
  for (int j = threadIdx.x; j < len; j += blockDim.x)
    starts[base + j] = (uint16_t)(row[j] << sh);
}

// Largest j in [0, nb) with row[j] << sh <= v (row strictly increasing,
// row[0] = 0).
__device__ __forceinline__ int bucket_of(const int32_t *row, int nb, int v, uint32_t sh) {
  int lo = 0, hi = nb - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if ((row[mid] << sh) <= v) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// A slot-filling launch counts its bitmap words and search flag in the
// build words of the table set's header (zero between launches); its last
// block to finish publishes them in the words the coders read
// (kChunkUsedWord, kSearchFlagWord) and clears the build words, so no launch
// needs a reset before it.
constexpr uint32_t kBuildUsedWord = 18;    // bitmap words handed out so far
constexpr uint32_t kBuildSearchWord = 19;  // 1 once a slot of the launch searches
constexpr uint32_t kBuildDoneWord = 20;    // blocks of the launch that have finished
// The Gaussian multiplier m = -Phi^-1(tail / 2) of the last scale-table
// refresh and its tail, two doubles (words 22-23 and 24-25; zero after
// prepare, which no valid tail matches): the next refresh with the same tail
// reads m instead of evaluating the inverse CDF in every block.
constexpr uint32_t kTailKeyWord = 22;
constexpr uint32_t kMultWord = 24;

// Where a table set's bitmap words go: they follow the slots of all rows.
struct ChunkArea {
  uint32_t base;  // slot-word index of the first bitmap word
  uint32_t cap;   // bitmap words available
  uint32_t *hdr;  // the table set's header words (the build words)
};

// Ends a slot-filling launch: every thread of every block calls it once,
// after its last bitmap allocation.  The build words are only touched by
// atomics; the block barrier orders every thread's build-word atomics before
// thread 0's increment of the done counter, whose release (with the barrier)
// makes them visible to the block that acquires the last increment.  That block
// publishes the build's bitmap count and search flag and clears the build
// words for the next launch.  (No thread waits for its slot stores here:
// only the next launch reads them.)
// With `tail` in (0, 1) the last block also caches the multiplier `mult` of
// that tail (every block has read the cache before it arrives).
__device__ void finish_build(const ChunkArea &ca, double tail = 0.0, double mult = 0.0) {
  __syncthreads();
  if (threadIdx.x != 0) return;
  const uint32_t blocks = gridDim.x * gridDim.y * gridDim.z;
  uint32_t done;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;"
               : "=r"(done)
               : "l"(ca.hdr + kBuildDoneWord)
               : "memory");
  if (done != blocks - 1) return;
  if (tail > 0.0 && tail < 1.0) {
    double *hd = reinterpret_cast<double *>(ca.hdr);
    hd[kTailKeyWord / 2] = tail;
    hd[kMultWord / 2] = mult;
  }
  // both build words read and cleared in one round trip
  uint32_t used, search;
  asm volatile(
      "atom.relaxed.gpu.global.exch.b32 %0, [%2], 0;\n\t"
      "atom.relaxed.gpu.global.exch.b32 %1, [%3], 0;"
      : "=r"(used), "=r"(search)
      : "l"(ca.hdr + kBuildUsedWord), "l"(ca.hdr + kBuildSearchWord)
      : "memory");
  ca.hdr[kChunkUsedWord] = used;
  ca.hdr[kSearchFlagWord] = search;
  ca.hdr[kBuildDoneWord] = 0u;
}

// Slots are filled kSlotsPerThread consecutive ones per thread, each from
// two binary searches (the buckets holding its first and last cumulative
// values), so no thread's work depends on how the buckets fall.  A block
// covers kSlotsPerBlock slots of one row and stages the row in shared
// memory when it has at most kRowSmem entries.
constexpr int kSlotThreads = 256;
constexpr int kSlotsPerThread = 1;
constexpr int kSlotsPerBlock = kSlotThreads * kSlotsPerThread;
constexpr int kRowSmem = 8192;
constexpr uint32_t kSlotSmemBytes = 4u * kRowSmem;

// The bitmap word of the 16 cumulative values [c0, c0 + 16) cut to [c0, c1),
// given jj, the bucket holding c0: bit i marks a bucket starting at c0 + i.
// The row is strictly increasing, so the buckets starting inside are
// jj + 1 .. jj + 15 at most and their loads do not wait on one another.
__device__ __forceinline__ uint32_t boundary_bits(const int32_t *row, int nb, int jj, int c0,
                                                  int c1, uint32_t sh) {
  uint32_t bits = 0;
#pragma unroll
  for (int u = 1; u <= 15; ++u) {
    const int i = jj + u;
    const int v = i < nb ? row[i] << sh : (int)kTotal;
    if (v < c1) bits |= 1u << ((v - c0) & 31);
  }
  return bits;
}

// The slots [tb, tb + kSlotsPerBlock) of a row (row in shared or global
// memory, entries scaled by << sh).
// SPT slots per thread, blockDim.x apart (so that a warp's stores stay
// coalesced), their searches independent of one another.
// LO: lo_tab holds the bucket of every slot's first value (slot_lo_table),
// else each slot searches the row for it.
template <int SPT = kSlotsPerThread, bool LO = false>
__device__ void fill_slot_block(const int32_t *row, int nb, uint32_t slot0, int w, int nslots,
                                int tb, uint32_t *slots, const ChunkArea &ca, uint32_t sh,
                                const uint16_t *lo_tab = nullptr) {
  const int lane = threadIdx.x & 31;
  const int t0 = tb + (int)threadIdx.x;
  const uint32_t nch = w > 16 ? (uint32_t)(w >> 4) : 1u;  // bitmap words of a slot
  int lo[SPT], hi[SPT];
  uint32_t need = 0;
  // lo: the bucket holding the slot's first value, one search per slot;
  // hi, the bucket holding its last value, is the next slot's lo (the next
  // lane's), less one when a bucket starts exactly at the next slot
#pragma unroll
  for (int u = 0; u < SPT; ++u) {
    const int t = t0 + u * (int)blockDim.x;
    lo[u] = t < nslots ? (LO ? (int)lo_tab[t] : bucket_of(row, nb, t * w, sh)) : 0;
  }
#pragma unroll
  for (int u = 0; u < SPT; ++u) {
    const int t = t0 + u * (int)blockDim.x;
    int next = __shfl_down_sync(kFull, lo[u], 1);
    if (lane == 31 && t + 1 < nslots)
      next = LO ? (int)lo_tab[t + 1] : bucket_of(row, nb, (t + 1) * w, sh);
    hi[u] = 0;
    if (t < nslots) {
      hi[u] = t + 1 >= nslots ? nb - 1 : ((row[next] << sh) == (t + 1) * w ? next - 1 : next);
      if (hi[u] - lo[u] >= 3) need += nch;
    }
  }
  // bitmap words: one allocation per warp
  uint32_t incl = need;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += v;
  }
  const uint32_t wtot = __shfl_sync(kFull, incl, 31);
  uint32_t wbase = 0;
  if (lane == 31 && wtot > 0) wbase = atomicAdd(ca.hdr + kBuildUsedWord, wtot);
  uint32_t at = __shfl_sync(kFull, wbase, 31) + incl - need;
#pragma unroll
  for (int u = 0; u < SPT; ++u) {
    const int t = t0 + u * (int)blockDim.x;
    if (t >= nslots) continue;
    const int a = t * w;
    const int inside = hi[u] - lo[u];
    uint32_t word;
    if (inside <= 2) {
      uint32_t e1 = 255u, e2 = 255u;
      if (inside >= 1) e1 = (uint32_t)((row[lo[u] + 1] << sh) - a - 1);
      if (inside == 2) e2 = (uint32_t)((row[lo[u] + 2] << sh) - a - 1);
      word = (uint32_t)lo[u] | (e1 << 16) | (e2 << 24);
    } else {
      if (at <= ca.cap && nch <= ca.cap - at && ca.base + at + nch <= kMaxChunkIndex) {
        const uint32_t p = ca.base + at;
        int jj = lo[u];  // bucket holding the word's first value
        for (uint32_t k = 0; k < nch; ++k) {
          const int c0 = a + 16 * (int)k;
          const int c1 = c0 + 16 < a + w ? c0 + 16 : a + w;
          const uint32_t bits = boundary_bits(row, nb, jj, c0, c1, sh);
          slots[p + k] = bits | ((uint32_t)jj << 16);
          // the bucket holding c0 + 16: past the boundaries inside, and one
          // more if a bucket starts exactly there
          jj += __popc(bits);
          if (jj + 1 < nb && (row[jj + 1] << sh) == c0 + 16) ++jj;
        }
        word = (p & 0xffffu) | (255u << 16) | ((p >> 16) << 24);
      } else {
        atomicExch(ca.hdr + kBuildSearchWord, 1u);
        const uint32_t e2 = (uint32_t)(inside - 3);
        word = (uint32_t)lo[u] | ((e2 + 1u) << 16) | (e2 << 24);
      }
      at += nch;
    }
    slots[slot0 + t] = word;
  }
}

// The bucket holding each slot's first value, for all 2^(16 - shift) slots of
// a row with nb buckets (entries scaled by << sh, strictly increasing, row[0]
// = 0 and row[nb] << sh = 65536), into lo_tab: bucket j holds the slots t
// with row[j] <= t * 2^shift < row[j + 1], so the buckets hand out every slot
// exactly once.  Every thread of the block calls it (it ends on a barrier).
__device__ __forceinline__ void slot_lo_table(const int32_t *row, int nb, int shift,
                                              uint16_t *lo_tab, uint32_t sh) {
  const int w1 = (1 << shift) - 1;
  for (int j = threadIdx.x; j < nb; j += blockDim.x) {
    const int te = ((row[j + 1] << sh) + w1) >> shift;
    for (int t = ((row[j] << sh) + w1) >> shift; t < te; ++t) lo_tab[t] = (uint16_t)j;
  }
  __syncthreads();
}

// Copies n row entries into shared memory with cp.async (every copy in
// flight at once, one wait), then a block barrier.
__device__ __forceinline__ void stage_row(int32_t *srow, const int32_t *grow, int n) {
  for (int i = threadIdx.x; i < n; i += blockDim.x) cp_async4(srow + i, grow + i);
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();
}

// Slot words (and bitmap words) of a row with nb buckets, blocks x, x +
// gridDim.x, ... of kSlotsPerBlock slots; grow[0..nb] is the row (grow[0] =
// 0, grow[nb] << sh = 65536), shift the row's slot width log2.  Every thread
// of the block must call it.
__device__ void fill_row_slots(const int32_t *grow, int nb, uint32_t slot0, int shift,
                               uint32_t *slots, const ChunkArea &ca, int32_t *srow,
                               uint32_t sh) {
  const int nslots = 1 << (16 - shift);
  const int w = 1 << shift;
  if ((int)blockIdx.x * kSlotsPerBlock >= nslots) return;  // (the whole block)
  const int32_t *row = grow;
  if (nb + 1 <= kRowSmem) {
    stage_row(srow, grow, nb + 1);
    row = srow;
  }
  for (int tb = blockIdx.x * kSlotsPerBlock; tb < nslots; tb += gridDim.x * kSlotsPerBlock)
    fill_slot_block(row, nb, slot0, w, nslots, tb, slots, ca, sh);
}

// Row r's packed buckets and 16-bit starts from its len entries (row[0] = 0
// and row[len - 1] << sh = 65536 checked by the caller); a bucket that is
// not strictly increasing or out of range records RANS_ERR_TABLE.
// With row_out, the row's entries are also copied there.
__device__ __forceinline__ void pack_row(const int32_t *row, int len, uint32_t base,
                                         uint32_t sh, uint32_t *buckets, uint16_t *starts,
                                         int32_t *status, int r, int32_t *row_out = nullptr) {
  const int32_t top = (int32_t)(kTotal >> sh);
  for (int j = threadIdx.x; j < len - 1; j += blockDim.x) {
    const int32_t a = row[j], b = row[j + 1];
    if (!(b > a) || a < 0 || b > top) {
      report(status, RANS_ERR_TABLE, r);
      continue;
    }
    buckets[base + j] = bucket_word(a, b, sh);
  }
  for (int j = threadIdx.x; j < len; j += blockDim.x) {
    const int32_t v = row[j];
    starts[base + j] = (uint16_t)(v << sh);
    if (row_out) row_out[j] = v;
  }
}

// Rebuilds a prepared table set from new CDF rows with the same lengths:
// block (x, r) fills slot block x of row r; block (0, r) also checks the
// row's length against the layout, refreshes its offset and packs its
// buckets.  Errors go to the blob's status word.
__global__ void __launch_bounds__(kSlotThreads)
    refresh_kernel(const int32_t *cdfs, int Lmax, const int32_t *lengths,
                   const int32_t *offsets, uint32_t sh, RowMeta *meta, uint32_t *buckets,
                   uint16_t *starts, uint32_t *slots, ChunkArea ca, int32_t *status) {
  extern __shared__ int32_t srow[];
  const int r = blockIdx.y;
  const RowMeta m = meta[r * kMetaCopies];
  const int len = lengths[r];
  const int32_t *row = cdfs + (size_t)r * (size_t)Lmax;
  const int32_t top = (int32_t)(kTotal >> sh);
  // (the conditions are the same on every thread of the block)
  if (len != (int)m.maxv + 2 || row[0] != 0 || row[len - 1] != top) {
    if (threadIdx.x == 0 && blockIdx.x == 0) report(status, RANS_ERR_TABLE, r);
  } else {
    if (blockIdx.x == 0) {
      const int32_t *prow = row;
      if (len <= kRowSmem) {
        stage_row(srow, row, len);
        prow = srow;
      }
      if (threadIdx.x < kMetaCopies) meta[r * kMetaCopies + threadIdx.x].offset = offsets[r];
      pack_row(prow, len, m.bucket_base, sh, buckets, starts, status, r);
      __syncthreads();  // the staged row is staged again below
    }
    fill_row_slots(row, len - 1, slot_base(m.slot), (int)slot_shift(m.slot), slots, ca, srow, sh);
  }
  finish_build(ca);
}

// The slot fill of rans_tables_prepare (rows already validated by
// pack_buckets_kernel; a malformed row only leaves its own slots undefined).
__global__ void __launch_bounds__(kSlotThreads)
    fill_slots_kernel(const int32_t *cdfs, int Lmax, const RowMeta *meta,
                      const int32_t *lengths, uint32_t sh, uint32_t *slots, ChunkArea ca) {
  extern __shared__ int32_t srow[];
  const int r = blockIdx.y;
  const RowMeta m = meta[r * kMetaCopies];
  const int32_t *row = cdfs + (size_t)r * (size_t)Lmax;
  const int len = lengths[r];
  if (len >= 2 && row[0] == 0 && row[len - 1] == (int32_t)(kTotal >> sh))
    fill_row_slots(row, len - 1, slot_base(m.slot), (int)slot_shift(m.slot), slots, ca, srow, sh);
  finish_build(ca);
}

// rans_build_cdfs_from_scales and rans_tables_refresh in one launch: block r
// quantises Gaussian row r as gaussian_rows_kernel does, then rewrites the
// row's offset, packed buckets, starts and every lookup slot of the row as
// refresh_kernel does, from the row it has just written (in shared memory
// when it fits).  A row that cannot be built, or whose length differs from the
// prepared layout, records RANS_ERR_TABLE in the blob's status word.
__global__ void __launch_bounds__(kRowThreads)
    gaussian_refresh_kernel(const float *scales, double tail, int prec, int32_t *cdfs, int Lmax,
                            int32_t *lengths, int32_t *offsets, RowMeta *meta, uint32_t *buckets,
                            uint16_t *starts, uint32_t *slots, ChunkArea ca, int32_t *status) {
  extern __shared__ __align__(16) double utab[];
  __shared__ BlockScratch sh;
  __shared__ QuantScratch qs;
  int32_t *rbuf = reinterpret_cast<int32_t *>(utab + kUTabBytes / 8);
  const int r = blockIdx.x;
  int32_t *row = cdfs + (size_t)r * (size_t)Lmax;
  // the multiplier cached by the last refresh, when it had this tail
  const double *hd = reinterpret_cast<const double *>(ca.hdr);
  const double mult = hd[kTailKeyWord / 2] == tail ? hd[kMultWord / 2] : gaussian_multiplier(tail);
  int32_t c = 0;
  int st = gaussian_center_m(scales[r], tail, mult, &c);
  const int len = 2 * c + 3;
  if (st == RANS_OK && len > Lmax) st = RANS_ERR_CAPACITY;
  // the row is quantised in shared memory when it fits, and packed, written
  // out and sliced from there
  int32_t *work = len <= kRowBufEntries ? rbuf : row;
  if (st == RANS_OK) {
    const double sd = (double)scales[r];
    const double *U = gauss_u_table(utab, (int)(kUTabBytes / 8), c, sd);
    GaussPmf pf{c, 2 * c + 1, sd, 1u << prec, U};
    st = quantise_row(pf, 2 * c + 2, work, sh, qs, 1u << prec);
  }
  for (int j = (st == RANS_OK ? len : 0) + threadIdx.x; j < Lmax; j += kRowThreads) row[j] = 0;
  if (threadIdx.x == 0) {
    lengths[r] = st ? st : len;
    offsets[r] = st ? 0 : -c;
  }
  // (st is the same on every thread)
  const RowMeta m = meta[r * kMetaCopies];
  if (st != RANS_OK || len != (int)m.maxv + 2) {
    if (st == RANS_OK && work != row) write_row(row, work, len);
    if (threadIdx.x == 0) report(status, RANS_ERR_TABLE, r);
  } else {
    const uint32_t ssh = (uint32_t)(kPrec - prec);
    // (quantise_row ends on a barrier: the row is complete)
    if (threadIdx.x < kMetaCopies) meta[r * kMetaCopies + threadIdx.x].offset = -c;
    pack_row(work, len, m.bucket_base, ssh, buckets, starts, status, r,
             work != row ? row : nullptr);
    const int shift = (int)slot_shift(m.slot);
    const int nslots = 1 << (16 - shift);
    if (work == rbuf) {
      // the slots' first buckets from the row's buckets, in the space of the
      // u table (2^14 slots at most)
      uint16_t *lo_tab = reinterpret_cast<uint16_t *>(utab);
      slot_lo_table(work, len - 1, shift, lo_tab, ssh);
      for (int tb = 0; tb < nslots; tb += kRowThreads * 4)
        fill_slot_block<4, true>(work, len - 1, slot_base(m.slot), 1 << shift, nslots, tb, slots,
                                 ca, ssh, lo_tab);
    } else {
      for (int tb = 0; tb < nslots; tb += kRowThreads * 4)
        fill_slot_block<4>(work, len - 1, slot_base(m.slot), 1 << shift, nslots, tb, slots, ca,
                           ssh);
    }
  }
  finish_build(ca, tail, mult);
}

// Alias tables, one row per block (the reading of the alias method given
// with RANS_FMT_ALIAS: Vose with first-in first-out worklists in ascending
// order, a symbol's own slot part ranked first and its alias parts after in
// slot order).  Thread 0 builds the slots (a short sequential pass over the
// row's n <= 8192 buckets, in shared memory); then every thread writes slot
// words and remap entries.
constexpr int kAliasMaxBuckets = 8192;

__global__ void __launch_bounds__(256)
    alias_build_kernel(const int32_t *cdfs, int Lmax, const int32_t *lengths,
                       const RowMeta *meta, int prec, int nmax, uint2 *aslots,
                       uint16_t *remap, int32_t *status) {
  extern __shared__ int32_t asm_[];
  __shared__ int ok_sh;
  const int r = blockIdx.x;
  const int n = lengths[r] - 1;
  const int32_t *row = cdfs + (size_t)r * (size_t)Lmax;
  const int32_t M = 1 << prec;
  int32_t *rem = asm_, *small = asm_ + nmax, *large = asm_ + 2 * nmax;
  int32_t *d = asm_ + 3 * nmax, *a = asm_ + 4 * nmax, *base = asm_ + 5 * nmax;
  if (threadIdx.x == 0) {
    int ok = n >= 1 && n <= nmax && (n & (n - 1)) == 0 && n <= M && row[0] == 0 && row[n] == M;
    const int32_t B = ok ? M / n : 1;
    int ns = 0, nl = 0, hs = 0, hl = 0;
    for (int j = 0; ok && j < n; ++j) {
      const int32_t f = row[j + 1] - row[j];
      if (f <= 0) {
        ok = 0;
        break;
      }
      rem[j] = f;
      d[j] = B;
      a[j] = j;
      base[j] = 0;
      if (f < B) small[ns++] = j;
      else if (f > B) large[nl++] = j;
    }
    while (ok && hs < ns && hl < nl) {
      const int32_t l = small[hs++];
      const int32_t g = large[hl];
      d[l] = rem[l];
      a[l] = g;
      rem[g] -= B - rem[l];
      if (rem[g] <= B) {
        ++hl;
        if (rem[g] < B) small[ns++] = g;
      }
    }
    if (ok && (hs < ns || hl < nl)) ok = 0;
    if (ok) {
      int32_t *cnt = rem;  // each symbol's next rank: own part first
      for (int j = 0; j < n; ++j) cnt[j] = d[j];
      for (int j = 0; j < n; ++j) {
        if (d[j] == B) continue;
        base[j] = cnt[a[j]];
        cnt[a[j]] += B - d[j];
      }
      // every symbol ends with exactly its frequency's positions, so the
      // remap writes below stay inside the row
      for (int j = 0; j < n; ++j)
        if (cnt[j] != row[j + 1] - row[j]) ok = 0;
    }
    if (!ok) report(status, RANS_ERR_TABLE, r);
    ok_sh = ok;
  }
  __syncthreads();
  if (!ok_sh) return;
  const uint32_t bb = meta[r * kMetaCopies].bucket_base;
  int log_b = 0;
  while ((n << log_b) < M) ++log_b;
  for (int j = threadIdx.x; j < n; j += blockDim.x)
    aslots[bb + j] = make_uint2((uint32_t)d[j], (uint32_t)a[j] | ((uint32_t)base[j] << 16));
  uint16_t *rm = remap + ((size_t)r << prec);
  for (int32_t c = threadIdx.x; c < M; c += blockDim.x) {
    const int32_t j = c >> log_b, o = c & ((1 << log_b) - 1);
    if (o < d[j]) rm[row[j] + o] = (uint16_t)c;
    else rm[row[a[j]] + base[j] + (o - d[j])] = (uint16_t)c;
  }
}

// Row index of every scale: through the key counts (ScaleKeys in
// rans_common.cuh) when the table qualifies, else by the search (scale_row).
__global__ void build_indexes_kernel(const float *scales, int64_t n, const float *table, int K,
                                     float bound, int32_t *indexes) {
  __shared__ float stab[64];
  __shared__ uint16_t cnt[kScaleKeyWords];
  ScaleKeys keys{};
  bool use_keys = false;
  if (K <= 64) {  // (uniform: every thread takes the same branch)
    for (int i = threadIdx.x; i < K; i += blockDim.x) stab[i] = table[i];
    __syncthreads();
    use_keys = build_scale_keys(stab, K, bound, cnt, keys);
  }
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float s = bound_scale(__ldg(scales + i), bound);
    indexes[i] = (int32_t)(use_keys ? keys.row(s) : scale_row(s, table, K));
  }
}

int ceil_log2(int64_t v) {
  int q = 0;
  while ((int64_t(1) << q) < v) ++q;
  return q;
}

}  // namespace

// ---- host entry points (called from api.cu) ------------------------------

int launch_gaussian_lengths(const float *scales, int K, double tail, int32_t *lengths,
                            int32_t *offsets, cudaStream_t st) {
  gaussian_lengths_kernel<<<(K + 127) / 128, 128, 0, st>>>(scales, K, tail, lengths, offsets);
  return cudaGetLastError() == cudaSuccess ? RANS_OK : RANS_ERR_CUDA;
}

int launch_gaussian_rows(const float *scales, int K, double tail, int prec, int32_t *cdfs,
                         int Lmax, int32_t *lengths, int32_t *offsets, cudaStream_t st) {
  if (ensure_dyn_smem((const void *)gaussian_rows_kernel, kGaussSmemBytes) != cudaSuccess)
    return RANS_ERR_CUDA;
  gaussian_rows_kernel<<<K, kRowThreads, kGaussSmemBytes, st>>>(scales, tail, prec, cdfs, Lmax,
                                                                lengths, offsets);
  return cudaGetLastError() == cudaSuccess ? RANS_OK : RANS_ERR_CUDA;
}

int launch_pmf_rows(const float *pmfs, int K, int stride, const int32_t *pmf_lengths,
                    const float *tail, int prec, int32_t *cdfs, int Lmax, int32_t *lengths,
                    cudaStream_t st) {
  pmf_rows_kernel<<<K, kRowThreads, kRowBufBytes, st>>>(pmfs, stride, pmf_lengths, tail, prec, cdfs, Lmax,
                                              lengths);
  return cudaGetLastError() == cudaSuccess ? RANS_OK : RANS_ERR_CUDA;
}

int launch_build_indexes(const float *scales, int64_t n, const float *scale_table, int32_t K,
                         float scale_bound, int32_t *indexes, cudaStream_t st) {
  if (n <= 0) return RANS_OK;
  int dev = 0;
  cudaGetDevice(&dev);
  int64_t blocks = (n + 255) / 256;
  const int64_t cap = 16LL * num_sms(dev);
  if (blocks > cap) blocks = cap;
  build_indexes_kernel<<<(unsigned)blocks, 256, 0, st>>>(scales, n, scale_table, K,
                                                         scale_bound, indexes);
  return cudaGetLastError() == cudaSuccess ? RANS_OK : RANS_ERR_CUDA;
}

int refresh_tables(const int32_t *cdfs, int K, int Lmax, const int32_t *lengths,
                   const int32_t *offsets, const rans_tables &t, cudaStream_t st) {
  if (K != t.K) return RANS_ERR_ARG;
  char *b = reinterpret_cast<char *>(t.blob);
  int32_t *status = reinterpret_cast<int32_t *>(b);
  RowMeta *dmeta = reinterpret_cast<RowMeta *>(b + kHeaderBytes);
  uint32_t *dbuckets = reinterpret_cast<uint32_t *>(b + kHeaderBytes + t.meta_bytes);
  uint16_t *dstarts =
      reinterpret_cast<uint16_t *>(b + kHeaderBytes + t.meta_bytes + t.bucket_bytes);
  uint32_t *dslots = reinterpret_cast<uint32_t *>(b + kHeaderBytes + t.meta_bytes +
                                                  t.bucket_bytes + t.start_bytes);
  ChunkArea ca;
  ca.base = (uint32_t)t.n_slots;
  ca.cap = t.slot_bytes / 4 - (uint32_t)t.n_slots;
  ca.hdr = reinterpret_cast<uint32_t *>(b);
  // blocks of kSlotsPerBlock slots, enough for the table's largest row
  // (blocks past a smaller row's slots return at once)
  const int qmax = t.max_slot_log2 >= kMinQ && t.max_slot_log2 <= kMaxQ ? t.max_slot_log2 : kMaxQ;
  dim3 grid((unsigned)(((1 << qmax) + kSlotsPerBlock - 1) / kSlotsPerBlock), (unsigned)K);
  refresh_kernel<<<grid, kSlotThreads, kSlotSmemBytes, st>>>(
      cdfs, Lmax, lengths, offsets, (uint32_t)(kPrec - t.precision), dmeta, dbuckets, dstarts,
      dslots, ca, status);
  return cudaGetLastError() == cudaSuccess ? RANS_OK : RANS_ERR_CUDA;
}

int refresh_tables_from_scales(const float *scales, int K, double tail, int32_t *cdfs, int Lmax,
                               int32_t *lengths, int32_t *offsets, const rans_tables &t,
                               cudaStream_t st) {
  if (K != t.K) return RANS_ERR_ARG;
  char *b = reinterpret_cast<char *>(t.blob);
  int32_t *status = reinterpret_cast<int32_t *>(b);
  RowMeta *dmeta = reinterpret_cast<RowMeta *>(b + kHeaderBytes);
  uint32_t *dbuckets = reinterpret_cast<uint32_t *>(b + kHeaderBytes + t.meta_bytes);
  uint16_t *dstarts =
      reinterpret_cast<uint16_t *>(b + kHeaderBytes + t.meta_bytes + t.bucket_bytes);
  uint32_t *dslots = reinterpret_cast<uint32_t *>(b + kHeaderBytes + t.meta_bytes +
                                                  t.bucket_bytes + t.start_bytes);
  ChunkArea ca;
  ca.base = (uint32_t)t.n_slots;
  ca.cap = t.slot_bytes / 4 - (uint32_t)t.n_slots;
  ca.hdr = reinterpret_cast<uint32_t *>(b);
  if (ensure_dyn_smem((const void *)gaussian_refresh_kernel, kGaussSmemBytes) != cudaSuccess)
    return RANS_ERR_CUDA;
  gaussian_refresh_kernel<<<K, kRowThreads, kGaussSmemBytes, st>>>(
      scales, tail, t.precision, cdfs, Lmax, lengths, offsets, dmeta, dbuckets, dstarts, dslots,
      ca, status);
  return cudaGetLastError() == cudaSuccess ? RANS_OK : RANS_ERR_CUDA;
}

// Room for the bucket words and starts (each row with up to 63 entries of
// bank skew), the slots of every row at the largest q, as many bitmap words
// again, and 256 KB (shared-memory tables plan up to
// a quarter of their slot room as bitmap words; tables read from global
// memory as many words as slots).
// The bitmap words a row's slots need at 2^q slots: max(1, w / 16) for each
// slot of width w = 2^(16-q) with three or more bucket boundaries strictly
// inside it (the rule of fill_slot_block), counted on the host from the row
// (entries scaled to 16 bits by << sh; entries out of range are skipped, the
// device rejects such rows).
uint64_t bitmap_words_needed(const int32_t *row, int nb, int q, uint32_t sh) {
  const int w = 1 << (16 - q);
  const uint64_t nch = w > 16 ? (uint64_t)(w >> 4) : 1ull;
  const int nslots = 1 << q;
  std::vector<uint8_t> inner(nslots, 0);
  for (int j = 1; j < nb; ++j) {
    const int64_t v = (int64_t)row[j] << sh;
    if (v <= 0 || v >= (int64_t)kTotal || v % w == 0) continue;
    uint8_t &c = inner[v / w];
    if (c < 3) ++c;
  }
  uint64_t n = 0;
  for (int t = 0; t < nslots; ++t)
    if (inner[t] >= 3) n += nch;
  return n;
}

uint64_t tables_bytes_bound(int K, int Lmax) {
  if (K <= 0 || Lmax < 2) return 0;
  const int64_t nb = (int64_t)Lmax - 1;
  int q = ceil_log2(nb);
  q = q < kMinQ ? kMinQ : (q > kMaxQ ? kMaxQ : q);
  const uint64_t nbp = (uint64_t)nb + 63;  // with the bank skew pad
  return (uint64_t)kHeaderBytes + pad16(16ull * kMetaCopies * K) + pad16(4ull * K * nbp) +
         pad16(2ull * K * nbp + 2) + pad16(8ull * K * (1ull << q)) + 262144ull;
}

int prepare_tables(const int32_t *cdfs, int K, int Lmax, const int32_t *lengths,
                   const int32_t *offsets, int prec, void *blob, uint64_t blob_bytes,
                   rans_tables *out, cudaStream_t st) {
  const uint32_t sh = (uint32_t)(kPrec - prec);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return RANS_ERR_CUDA;
  if (K > 65535) return RANS_ERR_ARG;  // one grid row per table row below
  std::vector<int32_t> len(K), off(K);
  if (cudaMemcpyAsync(len.data(), lengths, sizeof(int32_t) * K, cudaMemcpyDeviceToHost, st) !=
          cudaSuccess ||
      cudaMemcpyAsync(off.data(), offsets, sizeof(int32_t) * K, cudaMemcpyDeviceToHost, st) !=
          cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return RANS_ERR_CUDA;

  std::vector<RowMeta> meta(K);
  std::vector<int> q(K);
  uint64_t nbuckets = 0;
  int max_nb = 0;
  // Row bases are skewed across shared-memory banks: rows of equal length
  // would otherwise start in the same bank, and the lanes of a warp, each
  // reading the same position of its own row (the first probe of a row
  // search), would all hit it.  Each row takes the smallest pad (< 64
  // entries) that starts its 16-bit starts in the least-used bank so far.
  uint32_t bank_use[32] = {0};
  for (int r = 0; r < K; ++r) {
    if (len[r] < 0) return len[r];
    if (len[r] < 2 || len[r] > Lmax) return RANS_ERR_TABLE;
    const int nb = len[r] - 1;
    uint32_t pad = 0, best = UINT32_MAX;
    for (uint32_t p = 0; p < 64; ++p) {
      const uint32_t use = bank_use[((nbuckets + p) >> 1) & 31];
      if (use < best) {
        best = use;
        pad = p;
      }
    }
    nbuckets += pad;
    ++bank_use[(nbuckets >> 1) & 31];
    meta[r].bucket_base = (uint32_t)nbuckets;
    meta[r].maxv = (uint32_t)(len[r] - 2);
    meta[r].offset = off[r];
    nbuckets += (uint64_t)nb;
    if (nb > max_nb) max_nb = nb;
    const int qq = ceil_log2(nb);
    q[r] = qq < kMinQ ? kMinQ : (qq > kMaxQ ? kMaxQ : qq);
  }
  if (nbuckets > (1ull << 31)) return RANS_ERR_ARG;

  const uint32_t meta_bytes = (uint32_t)pad16(16ull * kMetaCopies * K);
  const uint32_t bucket_bytes = (uint32_t)pad16(4ull * nbuckets);
  const uint32_t start_bytes = (uint32_t)pad16(2ull * nbuckets + 2);
  int optin = 0;
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  const int64_t budget = (int64_t)optin - 1024;  // room for barriers and scratch
  auto slot_total = [&]() {
    uint64_t t = 0;
    for (int r = 0; r < K; ++r) t += 1ull << q[r];
    return t;
  };
  // encoder: bucket words in shared memory when they fit beside the rings,
  // else the 16-bit starts (with room for at least 4 warps' rings), else
  // global memory
  const int enc_mode = (int64_t)meta_bytes + bucket_bytes + kEncStageBytes <= budget ? 1
                       : ((int64_t)meta_bytes + start_bytes + kEncStageBytes / 6 <= budget ? 2
                                                                                          : 0);
  bool dec_smem = false;
  uint64_t chunk_words = 0;
  if ((int64_t)meta_bytes + start_bytes + kDecRingRoom <= budget) {
    const int64_t room = budget - meta_bytes - start_bytes - kDecRingRoom;
    // About one slot per bucket; halve the largest row's lookup until its
    // slots and the bitmap words they need (counted from the rows) fit the
    // room.  Bitmap words get all the room the slots leave.
    std::vector<int32_t> rows((size_t)K * (size_t)Lmax);
    if (cudaMemcpyAsync(rows.data(), cdfs, sizeof(int32_t) * rows.size(), cudaMemcpyDeviceToHost,
                        st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
      return RANS_ERR_CUDA;
    std::vector<uint64_t> words(K);
    for (int r = 0; r < K; ++r)
      words[r] = (1ull << q[r]) + bitmap_words_needed(&rows[(size_t)r * Lmax], len[r] - 1, q[r], sh);
    auto total = [&]() {
      uint64_t t = 0;
      for (int r = 0; r < K; ++r) t += words[r];
      return t;
    };
    while ((int64_t)pad16(4ull * total()) > room) {
      int best = -1;
      for (int r = 0; r < K; ++r)
        if (q[r] > kMinQ && (best < 0 || q[r] >= q[best])) best = r;
      if (best < 0) break;
      --q[best];
      words[best] = (1ull << q[best]) +
                    bitmap_words_needed(&rows[(size_t)best * Lmax], len[best] - 1, q[best], sh);
    }
    const int64_t left = room - (int64_t)pad16(4ull * slot_total());
    dec_smem = left >= 0;
    if (dec_smem) {
      // bitmap words: twice what these rows need (a refresh from other rows
      // of the same lengths may need more; slots that find none left
      // search) and at most the room left, so that small tables leave
      // shared memory to the decoders' per-warp rings
      uint64_t bits = 0;
      for (int r = 0; r < K; ++r) bits += words[r] - (1ull << q[r]);
      const uint64_t want = ((2 * bits + 256 + 3) / 4) * 4;
      chunk_words = std::min<uint64_t>((uint64_t)(left / 16) * 4, want);
    }
  }
  uint64_t sbase = 0;
  for (int r = 0; r < K; ++r) {
    meta[r].slot = (uint32_t)sbase | ((uint32_t)(16 - q[r]) << 27);
    sbase += 1ull << q[r];
  }
  if (sbase >= (1ull << 27)) return RANS_ERR_ARG;
  if (!dec_smem) chunk_words = sbase;
  const uint64_t base_need = (uint64_t)kHeaderBytes + meta_bytes + bucket_bytes + start_bytes +
                             pad16(4ull * sbase);
  if (blob == nullptr || blob_bytes < base_need) return RANS_ERR_CAPACITY;
  // a smaller blob gets fewer bitmap words (slots then search instead)
  if (base_need + 4ull * chunk_words > blob_bytes)
    chunk_words = ((blob_bytes - base_need) / 16) * 4;
  const uint32_t slot_bytes = (uint32_t)pad16(4ull * (sbase + chunk_words));
  const uint64_t need = (uint64_t)kHeaderBytes + meta_bytes + bucket_bytes + start_bytes + slot_bytes;
  if ((reinterpret_cast<uintptr_t>(blob) & 255) != 0) return RANS_ERR_ARG;

  char *b = reinterpret_cast<char *>(blob);
  int32_t *status = reinterpret_cast<int32_t *>(b);
  RowMeta *dmeta = reinterpret_cast<RowMeta *>(b + kHeaderBytes);
  uint32_t *dbuckets = reinterpret_cast<uint32_t *>(b + kHeaderBytes + meta_bytes);
  uint16_t *dstarts = reinterpret_cast<uint16_t *>(b + kHeaderBytes + meta_bytes + bucket_bytes);
  uint32_t *dslots =
      reinterpret_cast<uint32_t *>(b + kHeaderBytes + meta_bytes + bucket_bytes + start_bytes);
  if (cudaMemsetAsync(b, 0, kHeaderBytes, st) != cudaSuccess) return RANS_ERR_CUDA;
  std::vector<RowMeta> meta8((size_t)K * kMetaCopies);
  for (int r = 0; r < K; ++r)
    for (int c = 0; c < kMetaCopies; ++c) meta8[(size_t)r * kMetaCopies + c] = meta[r];
  if (cudaMemcpyAsync(dmeta, meta8.data(), sizeof(RowMeta) * meta8.size(),
                      cudaMemcpyHostToDevice, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return RANS_ERR_CUDA;
  if (cudaMemsetAsync(dstarts, 0, start_bytes, st) != cudaSuccess) return RANS_ERR_CUDA;
  pack_buckets_kernel<<<K, 256, 0, st>>>(cdfs, Lmax, dmeta, lengths, sh, dbuckets, dstarts,
                                         status);
  int maxslots = 0;
  for (int r = 0; r < K; ++r) maxslots = maxslots > (1 << q[r]) ? maxslots : (1 << q[r]);
  dim3 grid((maxslots + kSlotsPerBlock - 1) / kSlotsPerBlock, K);
  ChunkArea ca;
  ca.base = (uint32_t)sbase;
  ca.cap = (uint32_t)(slot_bytes / 4 - sbase);
  ca.hdr = reinterpret_cast<uint32_t *>(b);
  fill_slots_kernel<<<grid, kSlotThreads, kSlotSmemBytes, st>>>(cdfs, Lmax, dmeta, lengths, sh,
                                                                 dslots, ca);
  if (cudaGetLastError() != cudaSuccess) return RANS_ERR_CUDA;
  StatusWord sw;
  if (cudaMemcpyAsync(&sw, status, sizeof(sw), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return RANS_ERR_CUDA;
  if (sw.code != 0) return sw.code;

  out->blob = blob;
  out->blob_bytes = need;
  out->K = K;
  out->max_buckets = max_nb;
  out->n_buckets = (int64_t)nbuckets;
  out->n_slots = (int64_t)sbase;
  out->meta_bytes = meta_bytes;
  out->bucket_bytes = bucket_bytes;
  out->start_bytes = start_bytes;
  out->slot_bytes = slot_bytes;
  // decoder: metadata, starts and slots in shared memory when they fit, else
  // metadata and starts (each lookup searching its row), else global memory
  out->enc_in_smem = enc_mode;
  out->dec_in_smem =
      dec_smem ? 1 : ((int64_t)meta_bytes + start_bytes + kDecStageBytes <= budget ? 2 : 0);
  out->device = dev;
  out->precision = prec;
  int qmax = kMinQ;
  for (int r = 0; r < K; ++r) qmax = q[r] > qmax ? q[r] : qmax;
  out->max_slot_log2 = qmax;
  return RANS_OK;
}

int prepare_alias(const int32_t *cdfs, int K, int Lmax, const int32_t *lengths,
                  rans_tables &t, void *alias, uint64_t alias_bytes, cudaStream_t st) {
  if (K != t.K || alias == nullptr || (reinterpret_cast<uintptr_t>(alias) & 255) != 0)
    return RANS_ERR_ARG;
  const uint64_t slot_bytes = (8ull * (uint64_t)t.n_buckets + 255) & ~255ull;
  const uint64_t need = slot_bytes + 2ull * (uint64_t)K * (1ull << t.precision);
  if (alias_bytes < need) return RANS_ERR_CAPACITY;
  std::vector<int32_t> len(K);
  if (cudaMemcpyAsync(len.data(), lengths, sizeof(int32_t) * K, cudaMemcpyDeviceToHost, st) !=
          cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return RANS_ERR_CUDA;
  int nmax = 1;
  for (int r = 0; r < K; ++r) {
    const int n = len[r] - 1;
    if (n < 1 || (n & (n - 1)) != 0 || n > kAliasMaxBuckets) return RANS_ERR_ARG;
    nmax = n > nmax ? n : nmax;
  }
  char *b = reinterpret_cast<char *>(t.blob);
  int32_t *status = reinterpret_cast<int32_t *>(b);
  const RowMeta *dmeta = reinterpret_cast<const RowMeta *>(b + kHeaderBytes);
  uint2 *aslots = reinterpret_cast<uint2 *>(alias);
  uint16_t *remap = reinterpret_cast<uint16_t *>(reinterpret_cast<char *>(alias) + slot_bytes);
  const uint32_t smem = 6u * 4u * (uint32_t)nmax;
  if (ensure_dyn_smem((const void *)alias_build_kernel, (uint32_t)(smem)) != cudaSuccess)
    return RANS_ERR_CUDA;
  if (cudaMemsetAsync(alias, 0, slot_bytes, st) != cudaSuccess) return RANS_ERR_CUDA;
  alias_build_kernel<<<K, 256, smem, st>>>(cdfs, Lmax, lengths, dmeta, t.precision, nmax, aslots,
                                           remap, status);
  if (cudaGetLastError() != cudaSuccess) return RANS_ERR_CUDA;
  StatusWord sw;
  if (cudaMemcpyAsync(&sw, status, sizeof(sw), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return RANS_ERR_CUDA;
  if (sw.code != 0) return sw.code;
  t.alias = alias;
  t.alias_bytes = need;
  t.alias_remap_offset = slot_bytes;
  return RANS_OK;
}

}  // namespace rb
