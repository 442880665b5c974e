/*
 * Oracle for the LSCD SpMM path: a plain, slow, obviously correct CPU
 * restatement of what the GPU library computes.  TEST INFRASTRUCTURE ONLY:
 * only the tests, the smoke check and the benchmark's CPU-baseline leg may
 * load it.  It shares no code, header, table or helper with the CUDA path.
 *
 * Sources: the Flash-LLM paper review page ("Flash-LLM: Enabling
 * Cost-Effective and Highly-Efficient Large Generative Model Inference with
 * Unstructured Sparsity", xllm-io.github.io paper review):
 *   - section 3, "core formulas": C = A x B, A (M x K) sparse weights,
 *     B (K x N) dense features; compute intensity
 *     CI = 2MNK / ((MK + KN + MN) * sizeof(dtype)) <= N.
 *   - section 3, "sparse encoding format: Tiled-CSL": A is cut into tiles;
 *     every tile's nonzeros are stored together in NonZeros[], each as one
 *     32-bit word holding a 16-bit value and a 16-bit in-tile index;
 *     TileOffsets[] locates each tile; the stream is read with 128-bit loads.
 *   - section 5, "key implementation details" item 3: fp16 inputs, fp32
 *     accumulation.
 *
 * Readings where the pages are silent:
 *   R1 tiles are enumerated row-major over the tile grid: t = i*TK + j.
 *   R2 the in-tile index is row-major: loc = r*tile_k + c (r, c relative to
 *      the tile origin); ragged edge tiles keep the full tile_k row pitch.
 *   R3 word = value_bits | (loc << 16): value in the low half, which comes
 *      first in little-endian memory, matching the "[value | index]" order.
 *   R4 an entry is stored iff its 16-bit pattern is not 0x0000 (so -0.0,
 *      NaN, Inf and subnormals survive and decode is bit-exact).
 *   R5 inside a tile, words are in ascending loc.
 *   R6 each tile's list is padded to a multiple of 4 words (16 bytes, the
 *      128-bit load granule) with the sentinel 0xFFFF0000 (value +0, loc
 *      0xFFFF); tile area must be <= 65535 so the sentinel is never a loc.
 *   R7 TileOffsets is int32, num_tiles + 1 entries, in 32-bit words:
 *      off[0] = 0, off[t+1] = off[t] + roundup4(count_t).
 *   R8 B is K x N stored column-major ([N][K]); C is M x N column-major
 *      ([N][M]).
 *   R9 fp32/fp64 -> fp16 rounding is round-to-nearest-even, overflow to Inf.
 *   R10 word order v2 (optional, 64 x 64 tiles): the page's bank-aware
 *      reorder restated for the B200 kernel's swizzled dense tile; see
 *      ref_tcsl_reorder_banks.  Offsets, words and decode are unchanged.
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -shared -fPIC -pthread.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define REF_OK 0
#define REF_ERR_ARG 1
#define REF_ERR_CAPACITY 4
#define REF_ERR_CORRUPT 6

#define SENTINEL 0xFFFF0000u

/* ---- fp16 <-> fp64, written from the IEEE 754 binary16 definition ---- */

double ref_half_to_double(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1F;
    int m = h & 0x3FF;
    double v;
    if (e == 0) {
        v = ldexp((double)m, -24);               /* subnormal: m * 2^-24 */
    } else if (e == 31) {
        v = (m == 0) ? INFINITY : NAN;
    } else {
        v = ldexp((double)(1024 + m), e - 25);   /* (1.m) * 2^(e-15) */
    }
    return sign ? -v : v;
}

/* Round a double to the nearest binary16, ties to even.  The scaling by a
 * power of two is exact, so rint (which rounds to nearest-even in the default
 * mode) performs the only rounding. */
uint16_t ref_double_to_half(double x) {
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (isnan(x)) return (uint16_t)(sign | 0x7E00);
    if (isinf(a)) return (uint16_t)(sign | 0x7C00);
    if (a < ldexp(1.0, -14)) {                   /* subnormal range */
        double q = rint(a * ldexp(1.0, 24));     /* units of 2^-24 */
        return (uint16_t)(sign | (uint16_t)q);   /* q == 1024 is the min normal */
    }
    int e;
    frexp(a, &e);                                /* a in [2^(e-1), 2^e) */
    e -= 1;                                      /* a in [2^e, 2^(e+1)) */
    double q = rint(ldexp(a, 10 - e));           /* in [1024, 2048] */
    if (q == 2048.0) { q = 1024.0; e += 1; }
    if (e > 15) return (uint16_t)(sign | 0x7C00);
    return (uint16_t)(sign | (uint16_t)((e + 15) << 10) | (uint16_t)(q - 1024.0));
}

/* ---- compute intensity, section 3 "core formulas" ---- */
double ref_ci(double M, double K, double N, double sizeof_dtype) {
    return 2.0 * M * N * K / ((M * K + K * N + M * N) * sizeof_dtype);
}

/* ---- Tiled-CSL encoder ---- */

static int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

static int check_shape(int64_t M, int64_t K, int64_t tile_m, int64_t tile_k) {
    if (M < 0 || K < 0 || tile_m <= 0 || tile_k <= 0) return REF_ERR_ARG;
    if (tile_m * tile_k > 65535) return REF_ERR_ARG;
    return REF_OK;
}

/* Count pass: off[t+1] - off[t] = roundup4(count of nonzero bit patterns in
 * tile t); *nnz = total count without padding. */
int ref_tcsl_count(const uint16_t* A, int64_t M, int64_t K, int64_t tile_m, int64_t tile_k,
                   int32_t* off, int64_t* nnz) {
    int rc = check_shape(M, K, tile_m, tile_k);
    if (rc) return rc;
    int64_t TM = cdiv(M, tile_m), TK = cdiv(K, tile_k);
    int64_t total = 0, words = 0;
    off[0] = 0;
    for (int64_t i = 0; i < TM; ++i) {
        for (int64_t j = 0; j < TK; ++j) {
            int64_t cnt = 0;
            for (int64_t r = i * tile_m; r < (i + 1) * tile_m && r < M; ++r)
                for (int64_t c = j * tile_k; c < (j + 1) * tile_k && c < K; ++c)
                    if (A[r * K + c] != 0) ++cnt;
            total += cnt;
            words += (cnt + 3) / 4 * 4;
            if (words > INT32_MAX) return REF_ERR_CAPACITY;
            off[i * TK + j + 1] = (int32_t)words;
        }
    }
    *nnz = total;
    return REF_OK;
}

/* Fill pass: walk each tile in loc order (rows, then columns) and append one
 * word per stored entry; pad to the offset boundary with the sentinel. */
int ref_tcsl_fill(const uint16_t* A, int64_t M, int64_t K, int64_t tile_m, int64_t tile_k,
                  const int32_t* off, uint32_t* words) {
    int rc = check_shape(M, K, tile_m, tile_k);
    if (rc) return rc;
    int64_t TM = cdiv(M, tile_m), TK = cdiv(K, tile_k);
    for (int64_t i = 0; i < TM; ++i) {
        for (int64_t j = 0; j < TK; ++j) {
            int64_t t = i * TK + j;
            int64_t w = off[t], end = off[t + 1];
            for (int64_t r = 0; r < tile_m; ++r) {
                int64_t gr = i * tile_m + r;
                if (gr >= M) break;
                for (int64_t c = 0; c < tile_k; ++c) {
                    int64_t gc = j * tile_k + c;
                    if (gc >= K) break;
                    uint16_t v = A[gr * K + gc];
                    if (v == 0) continue;
                    if (w >= end) return REF_ERR_CAPACITY;
                    uint32_t loc = (uint32_t)(r * tile_k + c);
                    words[w++] = (uint32_t)v | (loc << 16);
                }
            }
            while (w < end) words[w++] = SENTINEL;
        }
    }
    return REF_OK;
}

/* Word order v2 (bank-balanced), for 64 x 64 tiles only.
 *
 * The page's ahead-of-time reordering (section 3, the bank-conflict-aware
 * reorder of each tile's NonZeros) exists so that a warp's stores of
 * consecutive words into the dense shared-memory tile hit distinct banks.
 * Its A100 rule targets a layout that sm_100a does not use; this is the same
 * idea for the layout the B200 kernel expands into: the value at loc sits at
 * byte swz(2*loc) of a 64-row x 128-byte tile with the 128-byte swizzle
 * swz(x) = x ^ ((x >> 3) & 0x70), so its bank is (swz(2*loc) >> 2) & 31.
 *
 * Rule: the tile's real words (first in ascending loc, as R5 leaves them) are
 * placed window by window, a window being 32 consecutive positions from the
 * tile start (the last one shorter).  At the start of each window the 32
 * banks are ranked by how many of the tile's words in them are still
 * unplaced (most first, ties to the lower bank); the window then takes the
 * next unplaced word (lowest loc) of each bank in that rank order, skipping
 * banks with none left, and goes round the ranking again while it has room.
 * Sentinel padding stays at the tile end.  Offsets, the set of words and the
 * decoded matrix are those of the ascending order. */
static uint32_t bank_of_loc(uint32_t loc) {
    uint32_t x = 2u * loc;
    uint32_t off = x ^ ((x >> 3) & 0x70u);
    return (off >> 2) & 31u;
}

int ref_tcsl_reorder_banks(const int32_t* off, uint32_t* words, int64_t num_tiles, int64_t tile_m,
                           int64_t tile_k) {
    if (tile_m != 64 || tile_k != 64 || num_tiles < 0) return REF_ERR_ARG;
    uint32_t (*list)[4096] = malloc(sizeof(uint32_t[32][4096]));
    uint32_t* out = malloc(sizeof(uint32_t) * 4096);
    if (!list || !out) { free(list); free(out); return REF_ERR_CAPACITY; }
    int cnt[32], taken[32];
    int rc = REF_OK;
    for (int64_t t = 0; t < num_tiles && rc == REF_OK; ++t) {
        int64_t b0 = off[t], e0 = off[t + 1];
        if (e0 - b0 > 4096) { rc = REF_ERR_CORRUPT; break; }
        for (int b = 0; b < 32; ++b) cnt[b] = taken[b] = 0;
        int64_t n = 0;
        for (int64_t w = b0; w < e0; ++w) {
            uint32_t word = words[w];
            if (word == SENTINEL) break;
            uint32_t loc = word >> 16;
            if (loc >= 4096) { rc = REF_ERR_CORRUPT; break; }
            uint32_t b = bank_of_loc(loc);
            list[b][cnt[b]++] = word;
            ++n;
        }
        if (rc != REF_OK) break;
        int64_t placed = 0;
        while (placed < n) {
            int64_t room = n - placed < 32 ? n - placed : 32;
            int order[32];
            for (int b = 0; b < 32; ++b) order[b] = b;
            /* rank banks by unplaced words, most first, ties to the lower bank (insertion sort) */
            for (int i = 1; i < 32; ++i) {
                int b = order[i], j = i;
                while (j > 0) {
                    int a = order[j - 1];
                    int ra = cnt[a] - taken[a], rb = cnt[b] - taken[b];
                    if (ra > rb || (ra == rb && a < b)) break;
                    order[j] = a;
                    --j;
                }
                order[j] = b;
            }
            while (room > 0) {
                for (int i = 0; i < 32 && room > 0; ++i) {
                    int b = order[i];
                    if (taken[b] < cnt[b]) {
                        out[placed++] = list[b][taken[b]++];
                        --room;
                    }
                }
            }
        }
        for (int64_t i = 0; i < n; ++i) words[b0 + i] = out[i];
    }
    free(list);
    free(out);
    return rc;
}

/* Decoder: zero-fill, then write each non-sentinel word's value at its loc.
 * Rejects a loc outside the tile or outside the matrix. */
int ref_tcsl_decode(const int32_t* off, const uint32_t* words, int64_t M, int64_t K,
                    int64_t tile_m, int64_t tile_k, uint16_t* A) {
    int rc = check_shape(M, K, tile_m, tile_k);
    if (rc) return rc;
    int64_t TM = cdiv(M, tile_m), TK = cdiv(K, tile_k);
    memset(A, 0, (size_t)(M * K) * sizeof(uint16_t));
    for (int64_t t = 0; t < TM * TK; ++t) {
        int64_t i = t / TK, j = t % TK;
        for (int64_t w = off[t]; w < off[t + 1]; ++w) {
            uint32_t word = words[w];
            uint32_t loc = word >> 16;
            if (loc == 0xFFFF) continue;
            int64_t r = loc / tile_k, c = loc % tile_k;
            int64_t gr = i * tile_m + r, gc = j * tile_k + c;
            if (r >= tile_m || gr >= M || gc >= K) return REF_ERR_CORRUPT;
            A[gr * K + gc] = (uint16_t)(word & 0xFFFF);
        }
    }
    return REF_OK;
}

/* ---- SpMM over the nonzero list, fp64 accumulation ----
 * C64[n][m] = sum over stored entries (m, k, a) of a * B[n][k], visited in
 * tile order then word order, i.e. ascending k for every row m.  Each fp16
 * product is exact in fp64.  absC64 (optional) gets sum |a * B[n][k]|, the
 * scale of the tolerance bound.  C16 (optional) = fp16_rne(C64). */

typedef struct {
    const int32_t* off; const uint32_t* words;
    int64_t M, K, tile_m, tile_k, N;
    const uint16_t* B;
    double* C64; double* absC64; uint16_t* C16;
    int64_t strip_begin, strip_end;
    int status;
} spmm_job;

static void spmm_strips(spmm_job* jb) {
    int64_t TK = cdiv(jb->K, jb->tile_k);
    double* bk = (double*)malloc(sizeof(double) * (size_t)(jb->N > 0 ? jb->N : 1));
    for (int64_t i = jb->strip_begin; i < jb->strip_end; ++i) {
        int64_t r0 = i * jb->tile_m;
        int64_t r1 = r0 + jb->tile_m < jb->M ? r0 + jb->tile_m : jb->M;
        for (int64_t n = 0; n < jb->N; ++n)
            for (int64_t m = r0; m < r1; ++m) {
                jb->C64[n * jb->M + m] = 0.0;
                if (jb->absC64) jb->absC64[n * jb->M + m] = 0.0;
            }
        for (int64_t j = 0; j < TK; ++j) {
            int64_t t = i * TK + j;
            for (int64_t w = jb->off[t]; w < jb->off[t + 1]; ++w) {
                uint32_t word = jb->words[w];
                uint32_t loc = word >> 16;
                if (loc == 0xFFFF) continue;
                int64_t r = loc / jb->tile_k, c = loc % jb->tile_k;
                int64_t m = r0 + r, k = j * jb->tile_k + c;
                if (r >= jb->tile_m || m >= jb->M || k >= jb->K) { jb->status = REF_ERR_CORRUPT; free(bk); return; }
                double a = ref_half_to_double((uint16_t)(word & 0xFFFF));
                for (int64_t n = 0; n < jb->N; ++n) bk[n] = ref_half_to_double(jb->B[n * jb->K + k]);
                for (int64_t n = 0; n < jb->N; ++n) {
                    double p = a * bk[n];
                    jb->C64[n * jb->M + m] += p;
                    if (jb->absC64) jb->absC64[n * jb->M + m] += fabs(p);
                }
            }
        }
        if (jb->C16)
            for (int64_t n = 0; n < jb->N; ++n)
                for (int64_t m = r0; m < r1; ++m)
                    jb->C16[n * jb->M + m] = ref_double_to_half(jb->C64[n * jb->M + m]);
    }
    free(bk);
}

static void* spmm_thread(void* p) { spmm_strips((spmm_job*)p); return NULL; }

int ref_spmm(const int32_t* off, const uint32_t* words, int64_t M, int64_t K, int64_t tile_m,
             int64_t tile_k, const uint16_t* B, int64_t N, double* C64, double* absC64,
             uint16_t* C16, int nthreads) {
    int rc = check_shape(M, K, tile_m, tile_k);
    if (rc) return rc;
    if (N < 0) return REF_ERR_ARG;
    int64_t TM = cdiv(M, tile_m);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > TM) nthreads = (int)(TM > 0 ? TM : 1);
    spmm_job* jobs = (spmm_job*)calloc((size_t)nthreads, sizeof(spmm_job));
    pthread_t* th = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
    for (int t = 0; t < nthreads; ++t) {
        spmm_job j = {off, words, M, K, tile_m, tile_k, N, B, C64, absC64, C16,
                      TM * t / nthreads, TM * (t + 1) / nthreads, REF_OK};
        jobs[t] = j;
    }
    for (int t = 1; t < nthreads; ++t) pthread_create(&th[t], NULL, spmm_thread, &jobs[t]);
    spmm_strips(&jobs[0]);
    for (int t = 1; t < nthreads; ++t) pthread_join(th[t], NULL);
    int status = REF_OK;
    for (int t = 0; t < nthreads; ++t) if (jobs[t].status) status = jobs[t].status;
    free(jobs); free(th);
    return status;
}

/* Selected outputs only: for each requested row m (any order), the full row
 * of C over all N, accumulated in the same order as ref_spmm.  Outputs are
 * [nrows][N]. */
int ref_spmm_rows(const int32_t* off, const uint32_t* words, int64_t M, int64_t K,
                  int64_t tile_m, int64_t tile_k, const uint16_t* B, int64_t N,
                  const int64_t* rows, int64_t nrows, double* C64, double* absC64) {
    int rc = check_shape(M, K, tile_m, tile_k);
    if (rc) return rc;
    int64_t TK = cdiv(K, tile_k);
    for (int64_t q = 0; q < nrows; ++q) {
        int64_t m = rows[q];
        if (m < 0 || m >= M) return REF_ERR_ARG;
        int64_t i = m / tile_m, r = m % tile_m;
        for (int64_t n = 0; n < N; ++n) { C64[q * N + n] = 0.0; if (absC64) absC64[q * N + n] = 0.0; }
        for (int64_t j = 0; j < TK; ++j) {
            int64_t t = i * TK + j;
            for (int64_t w = off[t]; w < off[t + 1]; ++w) {
                uint32_t word = words[w];
                uint32_t loc = word >> 16;
                if (loc == 0xFFFF) continue;
                if ((int64_t)(loc / tile_k) != r) continue;
                int64_t k = j * tile_k + loc % tile_k;
                if (k >= K) return REF_ERR_CORRUPT;
                double a = ref_half_to_double((uint16_t)(word & 0xFFFF));
                for (int64_t n = 0; n < N; ++n) {
                    double p = a * ref_half_to_double(B[n * K + k]);
                    C64[q * N + n] += p;
                    if (absC64) absC64[q * N + n] += fabs(p);
                }
            }
        }
    }
    return REF_OK;
}

/* Brute force over the dense matrix: every k, zeros included, ascending. */
void ref_dense(const uint16_t* A, const uint16_t* B, int64_t M, int64_t K, int64_t N, double* C64) {
    for (int64_t n = 0; n < N; ++n)
        for (int64_t m = 0; m < M; ++m) {
            double s = 0.0;
            for (int64_t k = 0; k < K; ++k)
                s += ref_half_to_double(A[m * K + k]) * ref_half_to_double(B[n * K + k]);
            C64[n * M + m] = s;
        }
}

/* Array forms of the conversions, for the tests. */
void ref_half_to_double_array(const uint16_t* h, double* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = ref_half_to_double(h[i]);
}
void ref_double_to_half_array(const double* x, uint16_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = ref_double_to_half(x[i]);
}
