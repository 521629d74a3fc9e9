/*
 * A plain C client of librans_b200 (no Python, no PyTorch): builds Gaussian
 * CDF rows from a scale table on the device, prepares the tables, encodes
 * seeded symbols (one row index per symbol) into 32-way interleaved streams,
 * decodes them and compares.  Prints "ok <bytes>" and exits 0 on success.
 * Compiled and run by tests/test_c_abi.py.
 */
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime.h>

#include "rans_b200.h"

#define CK(x)                                                            \
    do {                                                                 \
        int st_ = (int)(x);                                              \
        if (st_ != 0) {                                                  \
            fprintf(stderr, "%s:%d: status %d (%s)\n", __FILE__, __LINE__, \
                    st_, rans_status_string(st_));                       \
            return 1;                                                    \
        }                                                                \
    } while (0)
#define CU(x)                                                            \
    do {                                                                 \
        if ((x) != cudaSuccess) {                                        \
            fprintf(stderr, "%s:%d: CUDA error\n", __FILE__, __LINE__);  \
            return 1;                                                    \
        }                                                                \
    } while (0)

static uint64_t lcg(uint64_t *s)
{
    *s = *s * 6364136223846793005ull + 1442695040888963407ull;
    return *s >> 33;
}

static void *dev_alloc(size_t n)
{
    void *p = NULL;
    /* cudaMalloc returns 256-byte aligned memory */
    return cudaMalloc(&p, n ? n : 1) == cudaSuccess ? p : NULL;
}

int main(void)
{
    enum { K = 16, N = 300000, S = 37 };
    float h_scales[K];
    for (int k = 0; k < K; ++k) h_scales[k] = 0.2f * (float)(k + 1);
    float *scales = (float *)dev_alloc(sizeof h_scales);
    int32_t *lengths = (int32_t *)dev_alloc(K * sizeof(int32_t));
    int32_t *offsets = (int32_t *)dev_alloc(K * sizeof(int32_t));
    if (!scales || !lengths || !offsets) return 1;
    CU(cudaMemcpy(scales, h_scales, sizeof h_scales, cudaMemcpyHostToDevice));

    /* row lengths first, to size the rows */
    CK(rans_gaussian_lengths(scales, K, 1e-9, lengths, offsets, NULL));
    int32_t h_len[K];
    CU(cudaMemcpy(h_len, lengths, sizeof h_len, cudaMemcpyDeviceToHost));
    int32_t Lmax = 0;
    for (int k = 0; k < K; ++k) Lmax = h_len[k] > Lmax ? h_len[k] : Lmax;
    int32_t *cdfs = (int32_t *)dev_alloc((size_t)K * Lmax * sizeof(int32_t));
    if (!cdfs) return 1;
    CK(rans_build_cdfs_from_scales(scales, K, 1e-9, 16, cdfs, Lmax, lengths, offsets, NULL));

    rans_tables tables;
    memset(&tables, 0, sizeof tables);
    uint64_t tb = rans_tables_bytes(K, Lmax);
    void *blob = dev_alloc(tb);
    if (!blob) return 1;
    CK(rans_tables_prepare(cdfs, K, Lmax, lengths, offsets, 16, blob, tb, &tables, NULL));

    /* seeded symbols: mostly small, some far outside the rows (escapes) */
    int32_t *h_sym = (int32_t *)malloc(N * sizeof(int32_t));
    int32_t *h_idx = (int32_t *)malloc(N * sizeof(int32_t));
    int32_t *h_back = (int32_t *)malloc(N * sizeof(int32_t));
    if (!h_sym || !h_idx || !h_back) return 1;
    uint64_t seed = 12345;
    for (int i = 0; i < N; ++i) {
        h_idx[i] = (int32_t)(lcg(&seed) % K);
        int32_t v = (int32_t)(lcg(&seed) % 9) - 4;
        if (lcg(&seed) % 100 == 0) v = (int32_t)(lcg(&seed) % 200000) - 100000;
        h_sym[i] = v;
    }
    int32_t *sym = (int32_t *)dev_alloc(N * sizeof(int32_t));
    int32_t *idx = (int32_t *)dev_alloc(N * sizeof(int32_t));
    int32_t *back = (int32_t *)dev_alloc(N * sizeof(int32_t));
    if (!sym || !idx || !back) return 1;
    CU(cudaMemcpy(sym, h_sym, N * sizeof(int32_t), cudaMemcpyHostToDevice));
    CU(cudaMemcpy(idx, h_idx, N * sizeof(int32_t), cudaMemcpyHostToDevice));

    rans_chunking ch;
    memset(&ch, 0, sizeof ch);
    ch.kind = RANS_CHUNK_CONTIG;
    ch.interleave = 32;
    ch.n_streams = S;
    ch.index_block = 1;
    ch.format = RANS_FMT_RANS64;
    if (rans_num_streams(&ch, N) != S) return 1;

    uint64_t cap = rans_max_compressed_bytes(&ch, N);
    uint64_t ews = rans_encode_workspace_bytes(&ch, N);
    uint64_t dws = rans_decode_workspace_bytes(&ch, N);
    uint8_t *out = (uint8_t *)dev_alloc(cap);
    uint64_t *soff = (uint64_t *)dev_alloc((S + 1) * sizeof(uint64_t));
    void *enc_ws = dev_alloc(ews);
    void *dec_ws = dev_alloc(dws);
    if (!out || !soff || !enc_ws || !dec_ws) return 1;

    CK(rans_encode_with_indexes(sym, RANS_SYM_INT32, idx, N, &tables, &ch, out, cap, soff,
                                enc_ws, ews, NULL));
    CK(rans_get_status(enc_ws, NULL));
    uint64_t total = 0;
    CU(cudaMemcpy(&total, soff + S, sizeof total, cudaMemcpyDeviceToHost));

    CK(rans_decode_with_indexes(out, total, soff, idx, N, &tables, &ch, back, RANS_SYM_INT32,
                                dec_ws, dws, NULL));
    CK(rans_get_status(dec_ws, NULL));
    CU(cudaMemcpy(h_back, back, N * sizeof(int32_t), cudaMemcpyDeviceToHost));
    for (int i = 0; i < N; ++i) {
        if (h_back[i] != h_sym[i]) {
            fprintf(stderr, "mismatch at %d: %d != %d\n", i, h_back[i], h_sym[i]);
            return 1;
        }
    }
    /* a truncated container is reported, not mis-decoded silently */
    CK(rans_decode_with_indexes(out, total - 4, soff, idx, N, &tables, &ch, back,
                                RANS_SYM_INT32, dec_ws, dws, NULL));
    if (rans_get_status(dec_ws, NULL) == RANS_OK) {
        fprintf(stderr, "truncated container decoded without error\n");
        return 1;
    }
    printf("ok %llu\n", (unsigned long long)total);
    return 0;
}
