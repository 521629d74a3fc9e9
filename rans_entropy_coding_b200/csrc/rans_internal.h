// rans_internal.h -- host-side launchers shared between the librans_b200
// translation units (not part of the public ABI).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "rans_b200.h"

namespace rb {

struct Geom;

int launch_gaussian_lengths(const float *scales, int K, double tail, int32_t *lengths,
                            int32_t *offsets, cudaStream_t st);
// Rows summing to 2^prec (1 <= prec <= 16).
int launch_gaussian_rows(const float *scales, int K, double tail, int prec, int32_t *cdfs,
                         int Lmax, int32_t *lengths, int32_t *offsets, cudaStream_t st);
int launch_pmf_rows(const float *pmfs, int K, int stride, const int32_t *pmf_lengths,
                    const float *tail, int prec, int32_t *cdfs, int Lmax, int32_t *lengths,
                    cudaStream_t st);
uint64_t tables_bytes_bound(int K, int Lmax);
// Alias tables of a prepared table set into `alias` (synchronous).
int prepare_alias(const int32_t *cdfs, int K, int Lmax, const int32_t *lengths,
                  rans_tables &t, void *alias, uint64_t alias_bytes, cudaStream_t st);
int refresh_tables(const int32_t *cdfs, int K, int Lmax, const int32_t *lengths,
                   const int32_t *offsets, const rans_tables &t, cudaStream_t st);
// Gaussian rows (precision t.precision) into cdfs, lengths and offsets, and
// the prepared table set t rebuilt from them, in one launch.
int refresh_tables_from_scales(const float *scales, int K, double tail, int32_t *cdfs, int Lmax,
                               int32_t *lengths, int32_t *offsets, const rans_tables &t,
                               cudaStream_t st);
// Rows summing to 2^prec, stored scaled to 16 bits.
int prepare_tables(const int32_t *cdfs, int K, int Lmax, const int32_t *lengths,
                   const int32_t *offsets, int prec, void *blob, uint64_t blob_bytes,
                   rans_tables *out, cudaStream_t st);

// Encoder: codes every stream into its scratch slot and records its byte
// length in lens[S] (coder format g.fmt, rows of precision t.precision).
int launch_encode(const void *symbols, int sym_dtype, const int32_t *indexes,
                  const rans_tables &t, const Geom &g, char *scratch, uint64_t *lens,
                  int32_t *status, cudaStream_t st);
// Float latents in (one scale per element): rows from the scale table, symbols
// rint(y - mean); same outputs as launch_encode.
int launch_encode_float(const float *y, const float *means, const float *scales,
                        const float *scale_table, float scale_bound, const rans_tables &t,
                        const Geom &g, char *scratch, uint64_t *lens, int32_t *status,
                        cudaStream_t st);
// Compaction: exclusive scan of lens into offsets[S+1], then a copy of every
// stream from the end of its scratch slot to out + offsets[k].
int launch_compact(const Geom &g, const char *scratch, const uint64_t *lens, uint8_t *out,
                   uint64_t out_capacity, uint64_t *offsets, int32_t *status, cudaStream_t st);
// Float values out: float(symbol) + mean, rows from the scales.
int launch_decode_float(const uint8_t *in, uint64_t in_bytes, const uint64_t *offsets,
                        const float *scales, const float *means, const float *scale_table,
                        float scale_bound, const rans_tables &t, const Geom &g, float *values,
                        int32_t *status, cudaStream_t st);
// Row index of every scale (the float latents' rows), one thread per element.
int launch_build_indexes(const float *scales, int64_t n, const float *scale_table, int32_t K,
                         float scale_bound, int32_t *indexes, cudaStream_t st);
int launch_decode(const uint8_t *in, uint64_t in_bytes, const uint64_t *offsets,
                  const int32_t *indexes, const rans_tables &t, const Geom &g, void *symbols,
                  int sym_dtype, int32_t *status, cudaStream_t st);
int launch_debug_divide(const uint64_t *x, const uint32_t *f, int64_t n, uint64_t *q,
                        uint32_t *r, cudaStream_t st);

// A tensor map (CUtensorMap, 128 bytes, 64-byte aligned) for a 3-D int32
// tensor of width x height x depth elements (row-major, width fastest) and a
// box of box_w x box_h x 1; base 16-byte aligned, width * 4 a multiple of 16.
int encode_tile_map(void *map, const void *base, uint64_t width, uint64_t height,
                    uint64_t depth, uint32_t box_w, uint32_t box_h);

// Whether float latents (staged tensors a and b) can take the tile kernels.
bool flt_tile_shape_ok(const Geom &g, const void *a, const void *b);

// Device properties cached per device.
int num_sms(int device);
int smem_optin(int device);
// Kernel launch set-up, cached per (kernel, device): raise the kernel's
// dynamic shared memory limit to at least `bytes`, and its resident blocks
// per SM at `threads` threads and `smem` bytes of dynamic shared memory.
cudaError_t ensure_dyn_smem(const void *fn, uint32_t bytes);
cudaError_t blocks_per_sm(int *out, const void *fn, int threads, uint32_t smem);

}  // namespace rb
