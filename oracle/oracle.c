/*
 * oracle.c -- float64 CPU oracle for sequence-sharded paged decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code with
 * the CUDA path; its only shared input is the seeded generator header
 * synth/synth_hash.h, which holds no arithmetic of the method.
 *
 * Sources (web pages on Decode Context Parallelism):
 *  [blog]  "Efficient Decode Context Parallelism with vLLM for Long Context
 *          Workloads": section 4 (KV cache split by sequence position across
 *          GPUs), section 4.1 (AllGather Q -> local attention on the local KV
 *          slice -> partial output + LSE, merged with LSE weights, "the
 *          online-softmax trick"), section 5.3 (MLA: one latent shared by all
 *          query heads), section 5.4 (GQA: a KV head broadcast to its query
 *          heads).
 *  [guide] "Decode Context Parallel Guide" (vLLM Ascend), Constraints:
 *          cp_kv_cache_interleave_size sets the placement granularity.
 *
 * What is computed (plain definitions, float64):
 *  - ownership: position p of a request lives on shard (p / I) mod N, I the
 *    interleave size; a shard packs the positions it owns in increasing p, so
 *    the local index of p is (p / (I*N))*I + p mod I  (reading: the pages do
 *    not state the slot order; this is the plainest packing);
 *  - decode attention for one query row q (per head h, kv head g(h) =
 *    h / (Hq/Hkv)):  s_p = scale * q.k_p;  m = max s_p;  l = sum exp(s_p - m);
 *    O = sum exp(s_p - m) v_p / l;  LSE = m + ln l   (natural log);
 *    restricted to the positions a shard owns, this is that shard's partial;
 *    a shard owning no position gives O = 0, LSE = -inf;
 *  - merge: M = max_n LSE_n, LSE = M + ln sum_n exp(LSE_n - M),
 *    O = sum_n exp(LSE_n - LSE) O_n;
 *  - several query tokens per request (speculative decoding under DCP, blog
 *    section 6): with L_b positions, the QL new ones last, query token j
 *    attends the positions p <= L_b - QL + j (reading: the pages do not state
 *    the mask; this is the causal one);
 *  - MLA (absorbed form): key = the whole 576-wide latent row, value = its
 *    first Dv entries;
 *  - fp8 latent cache (e4m3, OCP "E4M3" with no infinities, max 448) with a
 *    per-token fp32 scale: scale = amax/448 (fp32), code = RNE(x/scale) with
 *    saturation to +-448; dequantised value = code * scale (exact in float64).
 *
 * Parity status of each function is recorded in the tests that pin it.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#include "../synth/synth_hash.h"

#define ORC_OK 0
#define ORC_ERR_ARG 1
#define ORC_ERR_UNALLOCATED 3

/* ------------------------------------------------------------------------ */
/* shard map                                                                 */
/* ------------------------------------------------------------------------ */

int32_t orc_owner(int64_t p, int32_t N, int32_t I) { return (int32_t)((p / I) % N); }

int64_t orc_local_index(int64_t p, int32_t N, int32_t I) {
    return (p / ((int64_t)I * N)) * I + (p % I);
}

/* number of positions in [0, L) owned by shard n */
int64_t orc_shard_count(int64_t L, int32_t N, int32_t I, int32_t n) {
    int64_t IN = (int64_t)I * N;
    int64_t full = (L / IN) * I;
    int64_t rem = L % IN - (int64_t)n * I;
    if (rem < 0) rem = 0;
    if (rem > I) rem = I;
    return full + rem;
}

void orc_shard_counts(int32_t B, const int64_t* seq_lens, int32_t N, int32_t I, int64_t* counts) {
    for (int32_t n = 0; n < N; n++)
        for (int32_t b = 0; b < B; b++) counts[(int64_t)n * B + b] = orc_shard_count(seq_lens[b], N, I, n);
}

/* For each (req[i], pos[i]): owner rank, local index, physical slot
 * bt[rank][req][local / P] * P + local % P, or -1 when that block-table entry
 * is not a page of the pool.  Returns ORC_ERR_UNALLOCATED if any slot is -1. */
int orc_shard_map(int64_t n_pos, const int32_t* pos, const int32_t* req, int32_t N, int32_t I,
                  int32_t P, const int32_t* bt, int32_t B, int32_t max_local_pages, int32_t num_pages,
                  int32_t* rank_out, int32_t* local_out, int64_t* slot_out) {
    if (N < 1 || I < 1 || P < 1 || B < 1 || max_local_pages < 1) return ORC_ERR_ARG;
    int status = ORC_OK;
    for (int64_t i = 0; i < n_pos; i++) {
        int64_t p = pos[i];
        int32_t b = req ? req[i] : (int32_t)i;
        int32_t r = orc_owner(p, N, I);
        int64_t l = orc_local_index(p, N, I);
        rank_out[i] = r;
        local_out[i] = (int32_t)l;
        int64_t j = l / P;
        int64_t page = -1;
        if (b >= 0 && b < B && j < max_local_pages)
            page = bt[((int64_t)r * B + b) * max_local_pages + j];
        if (page < 0 || page >= num_pages) {
            slot_out[i] = -1;
            status = ORC_ERR_UNALLOCATED;
        } else {
            slot_out[i] = page * P + (l % P);
        }
    }
    return status;
}

/* ------------------------------------------------------------------------ */
/* e4m3 (OCP 8-bit float, E4M3: bias 7, 3 mantissa bits, no inf, max 448)    */
/* ------------------------------------------------------------------------ */

double orc_e4m3_decode(uint8_t c) {
    int s = c >> 7, e = (c >> 3) & 0xF, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);           /* 2^-6 * m/8 */
    else v = ldexp(8.0 + m, e - 10);                 /* 2^(e-7) * (1 + m/8) */
    return s ? -v : v;
}

/* round-to-nearest-even onto the e4m3 grid, saturating finite values to +-448 */
uint8_t orc_e4m3_encode(double x) {
    uint8_t s = (x < 0 || (x == 0 && signbit(x))) ? 0x80 : 0;
    double a = fabs(x);
    if (isnan(x)) return 0x7F;
    if (a >= 448.0) return s | 0x7E;
    if (a == 0.0) return s;
    int e2;
    frexp(a, &e2);                  /* a = f * 2^e2, f in [0.5, 1): floor(log2 a) = e2 - 1 */
    int e = e2 - 1;
    if (e < -6) e = -6;             /* subnormal spacing below 2^-6 */
    double quantum = ldexp(1.0, e - 3);
    double k = a / quantum;         /* exact: division by a power of two */
    double fl = floor(k);
    double frac = k - fl;
    double r = fl;
    if (frac > 0.5 || (frac == 0.5 && fmod(fl, 2.0) != 0.0)) r = fl + 1.0;
    double v = r * quantum;
    if (v >= 448.0) return s | 0x7E;
    /* encode v */
    if (v < ldexp(1.0, -6)) return s | (uint8_t)(v / ldexp(1.0, -9));
    int ev2;
    frexp(v, &ev2);
    int ev = ev2 - 1;
    int m = (int)(v / ldexp(1.0, ev - 3)) - 8;
    return s | (uint8_t)(((ev + 7) << 3) | m);
}

/* Quantise one latent row (bf16 bits) to e4m3 codes and an fp32 scale. */
void orc_quantize_row_e4m3(const uint16_t* row_bf16, int32_t W, uint8_t* codes, float* scale_out) {
    float amax = 0.0f;
    for (int32_t d = 0; d < W; d++) {
        uint32_t u = (uint32_t)row_bf16[d] << 16;
        float x;
        memcpy(&x, &u, 4);
        float ax = fabsf(x);
        if (ax > amax) amax = ax;
    }
    if (amax == 0.0f) {
        *scale_out = 1.0f;
        memset(codes, 0, (size_t)W);
        return;
    }
    volatile float sc = amax / 448.0f;   /* single fp32 division, round to nearest */
    float scale = sc;
    for (int32_t d = 0; d < W; d++) {
        uint32_t u = (uint32_t)row_bf16[d] << 16;
        float x;
        memcpy(&x, &u, 4);
        volatile float y = x / scale;     /* single fp32 division, round to nearest */
        codes[d] = orc_e4m3_encode((double)y);
    }
    *scale_out = scale;
}

/* n rows of width W: codes [n][W], scales [n] */
void orc_quantize_rows_e4m3(int64_t n, int32_t W, const uint16_t* rows_bf16, uint8_t* codes, float* scales) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; i++) orc_quantize_row_e4m3(rows_bf16 + i * W, W, codes + i * W, scales + i);
}

/* ------------------------------------------------------------------------ */
/* decode attention                                                          */
/* ------------------------------------------------------------------------ */

typedef struct {
    int32_t kind;   /* 0 = GQA (separate K and V rows per kv head), 1 = MLA latent */
    int32_t fp8;    /* MLA only: latent stored as e4m3 codes + per-token fp32 scale */
    int32_t B, Hq, Hkv, Dk, Dv;
    double scale;
    /* row source: dense logical arrays (use_synth = 0) or the seeded generator */
    int32_t use_synth;
    const double* K;    /* [B][Lmax][Hkv][Dk]; MLA: latent rows [B][Lmax][Dk] */
    const double* V;    /* [B][Lmax][Hkv][Dv]; MLA: unused */
    int64_t Lmax;
    uint64_t seed;      /* value seed of the generator */
} orc_cache;

static double bf16_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* fetch the key row (Dk) or value row (Dv) of request b, position p, kv head g */
static void fetch_row(const orc_cache* c, int32_t b, int64_t p, int32_t g, int is_value, double* out,
                      uint16_t* tmp16, uint8_t* tmp8) {
    if (!c->use_synth) {
        if (c->kind == 1) {
            const double* row = c->K + ((int64_t)b * c->Lmax + p) * c->Dk;
            memcpy(out, row, sizeof(double) * (size_t)(is_value ? c->Dv : c->Dk));
        } else if (is_value) {
            memcpy(out, c->V + (((int64_t)b * c->Lmax + p) * c->Hkv + g) * c->Dv, sizeof(double) * (size_t)c->Dv);
        } else {
            memcpy(out, c->K + (((int64_t)b * c->Lmax + p) * c->Hkv + g) * c->Dk, sizeof(double) * (size_t)c->Dk);
        }
        return;
    }
    if (c->kind == 1) {
        uint64_t key = synth_key(c->seed, SYNTH_T_LATENT);
        int32_t W = c->Dk;
        for (int32_t d = 0; d < W; d++) tmp16[d] = synth_bf16_at(key, synth_kv_index(b, p, 0, d, 1, W));
        int32_t n = is_value ? c->Dv : c->Dk;
        if (c->fp8) {
            float sc;
            orc_quantize_row_e4m3(tmp16, W, tmp8, &sc);
            for (int32_t d = 0; d < n; d++) out[d] = orc_e4m3_decode(tmp8[d]) * (double)sc;
        } else {
            for (int32_t d = 0; d < n; d++) out[d] = bf16_to_double(tmp16[d]);
        }
        return;
    }
    int32_t W = is_value ? c->Dv : c->Dk;
    uint64_t key = synth_key(c->seed, is_value ? SYNTH_T_V : SYNTH_T_K);
    for (int32_t d = 0; d < W; d++)
        out[d] = bf16_to_double(synth_bf16_at(key, synth_kv_index(b, p, g, d, c->Hkv, W)));
}

/* One query row set of request b (qb: [Hq][Dk]; results Ob: [Hq][Dv], lseb: [Hq]), the query heads
 * h in [h0, h1) that all read kv head g.  Positions: all p < L, or (shard >= 0) only those owned
 * by `shard`. */
static void attend_group(const orc_cache* c, const double* qb, int32_t b, int64_t L, int32_t g, int32_t h0,
                         int32_t h1, int32_t N, int32_t I, int32_t shard, double* Ob, double* lseb) {
    int32_t nh = h1 - h0, Dk = c->Dk, Dv = c->Dv;
    int64_t nsel = 0;
    if (shard < 0) nsel = L;
    else nsel = orc_shard_count(L, N, I, shard);
    if (nsel == 0) {
        for (int32_t h = h0; h < h1; h++) {
            memset(Ob + (int64_t)h * Dv, 0, sizeof(double) * (size_t)Dv);
            lseb[h] = -INFINITY;
        }
        return;
    }
    double* S = (double*)malloc(sizeof(double) * (size_t)nsel * (size_t)nh);
    double* row = (double*)malloc(sizeof(double) * (size_t)(Dk > Dv ? Dk : Dv));
    uint16_t* t16 = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(Dk > Dv ? Dk : Dv));
    uint8_t* t8 = (uint8_t*)malloc((size_t)(Dk > Dv ? Dk : Dv));
    double* m = (double*)malloc(sizeof(double) * (size_t)nh);
    double* l = (double*)malloc(sizeof(double) * (size_t)nh);

    /* pass 1: scores s_p = scale * q . k_p, running maximum */
    for (int32_t j = 0; j < nh; j++) m[j] = -INFINITY;
    int64_t i = 0;
    for (int64_t p = 0; p < L; p++) {
        if (shard >= 0 && orc_owner(p, N, I) != shard) continue;
        fetch_row(c, b, p, g, 0, row, t16, t8);
        for (int32_t j = 0; j < nh; j++) {
            const double* qh = qb + (int64_t)(h0 + j) * Dk;
            double dot = 0.0;
            for (int32_t d = 0; d < Dk; d++) dot += qh[d] * row[d];
            double s = c->scale * dot;
            S[i * nh + j] = s;
            if (s > m[j]) m[j] = s;
        }
        i++;
    }
    /* pass 2: l = sum exp(s - m), O = sum exp(s - m) v / l */
    for (int32_t j = 0; j < nh; j++) {
        l[j] = 0.0;
        memset(Ob + (int64_t)(h0 + j) * Dv, 0, sizeof(double) * (size_t)Dv);
    }
    i = 0;
    for (int64_t p = 0; p < L; p++) {
        if (shard >= 0 && orc_owner(p, N, I) != shard) continue;
        fetch_row(c, b, p, g, 1, row, t16, t8);
        for (int32_t j = 0; j < nh; j++) {
            double w = exp(S[i * nh + j] - m[j]);
            l[j] += w;
            double* Oh = Ob + (int64_t)(h0 + j) * Dv;
            for (int32_t d = 0; d < Dv; d++) Oh[d] += w * row[d];
        }
        i++;
    }
    for (int32_t j = 0; j < nh; j++) {
        double* Oh = Ob + (int64_t)(h0 + j) * Dv;
        for (int32_t d = 0; d < Dv; d++) Oh[d] /= l[j];
        lseb[h0 + j] = m[j] + log(l[j]);
    }
    free(S); free(row); free(t16); free(t8); free(m); free(l);
}

/* Decode attention for the requests in req_list (all B if NULL).
 * q: [B][Hq][Dk] float64 (exact bf16 values); O: [B][Hq][Dv]; lse: [B][Hq].
 * shard < 0: unsharded full context; shard = n: shard n's partial under (N, I). */
int orc_decode(const orc_cache* c, const double* q, const int64_t* seq_lens, int32_t N, int32_t I,
               int32_t shard, const int32_t* req_list, int32_t n_req, double* O, double* lse) {
    if (c->B < 1 || c->Hq < 1 || c->Hkv < 1 || c->Hq % c->Hkv || c->Dk < 1 || c->Dv < 1) return ORC_ERR_ARG;
    if (c->kind == 1 && (c->Hkv != 1 || c->Dv > c->Dk)) return ORC_ERR_ARG;
    if (shard >= 0 && (N < 1 || I < 1 || shard >= N)) return ORC_ERR_ARG;
    if (!req_list) n_req = c->B;
    int32_t group = c->Hq / c->Hkv;
    /* task = (request, head block); MLA splits its heads into blocks of 16 */
    int32_t hb = (c->kind == 1) ? (c->Hq < 16 ? c->Hq : 16) : group;
    int32_t blocks = (c->Hq + hb - 1) / hb;
    int64_t ntask = (int64_t)n_req * blocks;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < ntask; t++) {
        int32_t r = (int32_t)(t / blocks), k = (int32_t)(t % blocks);
        int32_t b = req_list ? req_list[r] : r;
        int32_t h0 = k * hb, h1 = h0 + hb > c->Hq ? c->Hq : h0 + hb;
        int32_t g = (c->kind == 1) ? 0 : h0 / group;
        attend_group(c, q + (int64_t)b * c->Hq * c->Dk, b, seq_lens[b], g, h0, h1, N, I, shard,
                     O + (int64_t)b * c->Hq * c->Dv, lse + (int64_t)b * c->Hq);
    }
    return ORC_OK;
}

/* Decode with QL query tokens per request (speculative decoding / multi-token prediction
 * running under DCP: blog section 6).  Request b holds L_b positions, the QL new tokens
 * included: query token j sits at position L_b - QL + j and attends the positions up to
 * and including its own, p < L_b - QL + j + 1 (causal among the new tokens; reading: the
 * pages name the combination but not the mask, and this is the standard one).
 * q: [B][QL][Hq][Dk]; O: [B][QL][Hq][Dv]; lse: [B][QL][Hq].  Requires L_b >= QL.
 * shard < 0: unsharded; shard = n: shard n's partial under (N, I). */
int orc_decode_multi(const orc_cache* c, const double* q, const int64_t* seq_lens, int32_t QL, int32_t N,
                     int32_t I, int32_t shard, double* O, double* lse) {
    if (c->B < 1 || c->Hq < 1 || c->Hkv < 1 || c->Hq % c->Hkv || c->Dk < 1 || c->Dv < 1 || QL < 1) return ORC_ERR_ARG;
    if (c->kind == 1 && (c->Hkv != 1 || c->Dv > c->Dk)) return ORC_ERR_ARG;
    if (shard >= 0 && (N < 1 || I < 1 || shard >= N)) return ORC_ERR_ARG;
    for (int32_t b = 0; b < c->B; b++)
        if (seq_lens[b] < QL) return ORC_ERR_ARG;
    int32_t group = c->Hq / c->Hkv;
    int32_t hb = (c->kind == 1) ? (c->Hq < 16 ? c->Hq : 16) : group;
    int32_t blocks = (c->Hq + hb - 1) / hb;
    int64_t ntask = (int64_t)c->B * QL * blocks;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < ntask; t++) {
        int64_t bj = t / blocks;
        int32_t k = (int32_t)(t % blocks);
        int32_t b = (int32_t)(bj / QL), j = (int32_t)(bj % QL);
        int32_t h0 = k * hb, h1 = h0 + hb > c->Hq ? c->Hq : h0 + hb;
        int32_t g = (c->kind == 1) ? 0 : h0 / group;
        attend_group(c, q + bj * c->Hq * c->Dk, b, seq_lens[b] - QL + j + 1, g, h0, h1, N, I, shard,
                     O + bj * c->Hq * c->Dv, lse + bj * c->Hq);
    }
    return ORC_OK;
}

/* LSE-weighted merge of N partials: O_part [N][B][H][Dv], lse_part [N][B][H]. */
void orc_merge(int32_t N, int32_t B, int32_t H, int32_t Dv, const double* O_part, const double* lse_part,
               double* O, double* lse) {
    for (int64_t bh = 0; bh < (int64_t)B * H; bh++) {
        double M = -INFINITY;
        for (int32_t n = 0; n < N; n++) {
            double x = lse_part[(int64_t)n * B * H + bh];
            if (x > M) M = x;
        }
        double* o = O + bh * Dv;
        memset(o, 0, sizeof(double) * (size_t)Dv);
        if (M == -INFINITY) {
            lse[bh] = -INFINITY;
            continue;
        }
        double sum = 0.0;
        for (int32_t n = 0; n < N; n++) sum += exp(lse_part[(int64_t)n * B * H + bh] - M);
        double L = M + log(sum);
        lse[bh] = L;
        for (int32_t n = 0; n < N; n++) {
            double w = exp(lse_part[(int64_t)n * B * H + bh] - L);
            const double* on = O_part + ((int64_t)n * B * H + bh) * Dv;
            for (int32_t d = 0; d < Dv; d++) o[d] += w * on[d];
        }
    }
}

/* Generator values as the oracle sees them (for cross-checking the synth module):
 * out[i] = bf16 bits of stream key(seed, tensor) at indices idx[i]. */
void orc_synth_bf16(uint64_t seed, uint64_t tensor, int64_t n, const uint64_t* idx, uint16_t* out) {
    uint64_t key = synth_key(seed, tensor);
    for (int64_t i = 0; i < n; i++) out[i] = synth_bf16_at(key, idx[i]);
}

int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
