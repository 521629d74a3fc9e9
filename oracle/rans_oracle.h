/*
 * rans_oracle.h -- declarations of the CPU correctness oracle.
 *
 * TEST INFRASTRUCTURE ONLY: used by tests/, the smoke check and the bench's
 * CPU-baseline leg.  It is independent of the CUDA library and shares no
 * header with it.  All pointers are host pointers.  Status codes: 0 on
 * success, negative on error (the values below).
 */
#ifndef RANS_ORACLE_H
#define RANS_ORACLE_H

#include <stdint.h>

#define ORC_OK 0
#define ORC_ERR_ARG (-1)
#define ORC_ERR_INDEX (-2)
#define ORC_ERR_ZERO_FREQ (-3)
#define ORC_ERR_RANGE (-4)
#define ORC_ERR_CAPACITY (-5)
#define ORC_ERR_CORRUPT (-6)

#ifdef __cplusplus
extern "C" {
#endif

/* pmf (n entries, the last one the tail mass) -> cdf row of n + 1 entries. */
int orc_pmf_to_cdf(const float *pmf, int n, int32_t *cdf);

/* The same at precision prec (1..16): the row sums to 2^prec. */
int orc_pmf_to_cdf_prec(const float *pmf, int n, int prec, int32_t *cdf);

/* -Phi^-1(tail_mass / 2) by bisection on erfc. */
double orc_gaussian_multiplier(double tail_mass);
int orc_gaussian_center(float scale, double tail_mass, int32_t *center);

/* K Gaussian rows, each padded to Lmax int32 entries. */
int orc_build_cdfs_from_scales(const float *scales, int K, double tail_mass,
                               int32_t *cdfs, int Lmax, int32_t *lengths,
                               int32_t *offsets);

int orc_build_cdfs_from_scales_prec(const float *scales, int K, double tail_mass, int prec,
                                    int32_t *cdfs, int Lmax, int32_t *lengths,
                                    int32_t *offsets);

/* K rows from pmfs: row r is pmfs[r*stride .. r*stride + pmf_lengths[r]) plus
 * tail_mass[r]; cdf length pmf_lengths[r] + 2. */
int orc_build_cdfs_from_pmfs(const float *pmfs, int K, int stride,
                             const int32_t *pmf_lengths, const float *tail_mass,
                             int32_t *cdfs, int Lmax, int32_t *lengths);

int orc_build_cdfs_from_pmfs_prec(const float *pmfs, int K, int stride,
                                  const int32_t *pmf_lengths, const float *tail_mass,
                                  int prec, int32_t *cdfs, int Lmax, int32_t *lengths);

/* One stream of n symbols (in stream order) with their row indexes; W = 1, 2,
 * 4, 8 or 32 interleaved states.  Returns the byte length, or a negative status. */
int64_t orc_encode_stream(const int64_t *sym, const int32_t *row, int64_t n,
                          const int32_t *cdfs, int K, int Lmax,
                          const int32_t *lengths, const int32_t *offsets,
                          int W, uint8_t *out, int64_t cap);

/* Decodes n symbols of one stream of len bytes.  Returns a status. */
int orc_decode_stream(const uint8_t *in, int64_t len, const int32_t *row, int64_t n,
                      const int32_t *cdfs, int K, int Lmax,
                      const int32_t *lengths, const int32_t *offsets,
                      int W, int64_t *sym_out);

/* The rans32_16 variant: 32-bit state, 16-bit words, rows summing to 2^prec
 * (1 <= prec <= 15), W = 1, 2, 4, 8 or 32.  Byte lengths are even. */
int64_t orc_encode_stream16(const int64_t *sym, const int32_t *row, int64_t n,
                            const int32_t *cdfs, int K, int Lmax,
                            const int32_t *lengths, const int32_t *offsets,
                            int prec, int W, uint8_t *out, int64_t cap);
int orc_decode_stream16(const uint8_t *in, int64_t len, const int32_t *row, int64_t n,
                        const int32_t *cdfs, int K, int Lmax,
                        const int32_t *lengths, const int32_t *offsets,
                        int prec, int W, int64_t *sym_out);

/* Alias table of one row of len entries at precision prec (len - 1 a power
 * of two): per slot d, a, base (len - 1 entries each) and, unless NULL, the
 * 2^prec-entry remap. */
int orc_alias_build(const int32_t *cdf, int len, int prec, int32_t *d, int32_t *a,
                    int32_t *base, int32_t *remap);

/* Alias-coded streams: prec 16 = the 64-bit format, <= 15 = rans32_16;
 * W = 1, 2, 4 or 8. */
int64_t orc_encode_stream_alias(const int64_t *sym, const int32_t *row, int64_t n,
                                const int32_t *cdfs, int K, int Lmax,
                                const int32_t *lengths, const int32_t *offsets,
                                int prec, int W, uint8_t *out, int64_t cap);
int orc_decode_stream_alias(const uint8_t *in, int64_t len, const int32_t *row, int64_t n,
                            const int32_t *cdfs, int K, int Lmax,
                            const int32_t *lengths, const int32_t *offsets,
                            int prec, int W, int64_t *sym_out);

#ifdef __cplusplus
}
#endif

#endif
