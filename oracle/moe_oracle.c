/*
 * moe_oracle.c -- plain, slow CPU oracle for the single-GPU core of an
 * expert-parallel MoE layer (router top-k -> dispatch layout -> permute ->
 * grouped SwiGLU expert GEMM -> weighted combine).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the tests, the smoke check and the benchmark's CPU
 * baseline leg do.  It shares no code, header or table with the CUDA
 * library: every helper below (bf16 rounding, the FP8 e4m3 codec, the
 * softmax, the counting sort) is written here from its definition.
 *
 * Arithmetic is fp64 except where a value is defined by a narrower type:
 *   - router logits are compared as the fp32 values they are;
 *   - the FP8 payload's scale and quotient are fp32 IEEE divisions, because
 *     they decide an integer code (the quantised byte) and the CUDA side
 *     decides it in fp32 as well;
 *   - an operand the layer defines in a narrow type is rounded to it:
 *     the expert GEMMs take bf16 (or fp32) operands, so h is rounded to the
 *     weight dtype before the down projection;
 *   - everything else is exact: the results a caller compares (h, y, out)
 *     are returned unrounded in fp64 (dtype code 3), and combine sums y as
 *     given (fp64 y from the GEMM for the exact layer output); the router
 *     weights are returned in fp32, their storage type.
 *
 * Sources (page title, section):
 *   "Expert parallelism and all-to-all", "Walking through one MoE layer":
 *       route, dispatch, grouped expert matmul, weighted combine.
 *   "Expert Parallelism" (aiwiki), "Implementation": sort by destination
 *       (argsort), per-rank bincount, undo the sort after the experts.
 *   "Expert parallelism" (Transformers), "Adding an implementation" and
 *       "How the sizes combine": (hidden_states, top_k_index, top_k_weights)
 *       in, weighted expert output per token out; rank r owns experts
 *       [r*E/W, (r+1)*E/W).
 *   "Expert parallelism and all-to-all", "Traffic math": 1-byte FP8
 *       activation payload.
 *
 * dtype codes: 0 = fp32, 1 = bf16 (uint16 bits), 2 = FP8 e4m3 (OCP, "fn"),
 * 3 = fp64 (results only).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_F32 0
#define OR_BF16 1
#define OR_E4M3 2
#define OR_F64 3

/* ------------------------------------------------------------------ */
/* number formats, written from their definitions                      */
/* ------------------------------------------------------------------ */

/* Round a non-negative real r to the nearest integer, ties to even. */
static double rint_half_even(double r) {
    double n = floor(r);
    double f = r - n;
    if (f > 0.5) return n + 1.0;
    if (f < 0.5) return n;
    return (fmod(n, 2.0) == 0.0) ? n : n + 1.0;
}

/* bf16: 1 sign, 8 exponent (bias 127), 7 fraction bits; subnormal quantum
 * 2^-133; largest finite (2 - 2^-7) * 2^127.  Round-to-nearest-even from
 * the exact fp64 value. */
static uint16_t bf16_from_double(double v) {
    if (isnan(v)) return 0x7FC0;
    uint16_t s = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0) return s;
    if (isinf(a)) return s | 0x7F80;
    int e;
    frexp(a, &e);              /* a = f * 2^e, f in [0.5, 1): binade 2^(e-1) */
    int be = e - 1;
    double q = (be < -126) ? ldexp(1.0, -133) : ldexp(1.0, be - 7);
    double val = rint_half_even(a / q) * q;
    if (val > ldexp(255.0, 120)) return s | 0x7F80;  /* rounds past max: inf */
    float f = (float)val;      /* exact: val has <= 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, 4);
    return s | (uint16_t)((u >> 16) & 0x7FFF);
}

static double bf16_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* OCP 8-bit float E4M3 ("fn" variant): 1 sign, 4 exponent bits (bias 7),
 * 3 mantissa bits; no infinities; S.1111.111 is NaN; largest finite
 * S.1111.110 = 448; smallest normal 2^-6; subnormals m * 2^-9. */
static double e4m3_to_double(uint8_t c) {
    int E = (c >> 3) & 15, m = c & 7;
    if (E == 15 && m == 7) return NAN;
    double v = (E == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, E - 7);
    return (c & 0x80) ? -v : v;
}

/* Encode an fp32 value: round to nearest, ties to even, saturating
 * magnitudes above 448 to 448; NaN maps to 0x7F. */
static uint8_t e4m3_from_float(float v) {
    if (isnan(v)) return 0x7F;
    uint8_t s = signbit(v) ? 0x80 : 0;
    double a = fabs((double)v);
    if (a > 448.0) return s | 0x7E;
    double q;
    if (a < ldexp(1.0, -6)) {
        q = ldexp(1.0, -9);                    /* subnormal spacing */
    } else {
        int e;
        frexp(a, &e);
        q = ldexp(1.0, (e - 1) - 3);           /* 3 mantissa bits */
    }
    double val = rint_half_even(a / q) * q;    /* exact, <= 448 */
    if (val == 0.0) return s;
    if (val < ldexp(1.0, -6)) return s | (uint8_t)(val / ldexp(1.0, -9));
    int e;
    frexp(val, &e);
    int be = e - 1;                            /* val in [2^be, 2^(be+1)) */
    int m = (int)((val / ldexp(1.0, be) - 1.0) * 8.0);
    return s | (uint8_t)((be + 7) << 3) | (uint8_t)m;
}

static double load_elem(const void* base, int dt, int64_t i) {
    switch (dt) {
        case OR_F32: return (double)((const float*)base)[i];
        case OR_BF16: return bf16_to_double(((const uint16_t*)base)[i]);
        case OR_F64: return ((const double*)base)[i];
        default: return e4m3_to_double(((const uint8_t*)base)[i]);
    }
}

/* v rounded to storage type dt (fp32 or bf16), as a double */
static double round_to(int dt, double v) {
    return dt == OR_F32 ? (double)(float)v : bf16_to_double(bf16_from_double(v));
}

static void store_elem(void* base, int dt, int64_t i, double v) {
    if (dt == OR_F64) ((double*)base)[i] = v;
    else if (dt == OR_F32) ((float*)base)[i] = (float)v;
    else ((uint16_t*)base)[i] = bf16_from_double(v);
}

/* exported codec entry points (pinned by the CPU tests) */
void oracle_e4m3_encode(const float* v, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = e4m3_from_float(v[i]);
}
void oracle_e4m3_decode(const uint8_t* c, int64_t n, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = e4m3_to_double(c[i]);
}
void oracle_bf16_round(const double* v, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = bf16_from_double(v[i]);
}

/* ------------------------------------------------------------------ */
/* S1 route: top-k of the router logits + softmax over the k picks     */
/* ------------------------------------------------------------------ */
/* Experts are ordered by (logit descending, expert id ascending); the k
 * first ones are the picks, in that order.  The weights are the softmax
 * of the k picked logits, which equals the full softmax over E restricted
 * to the picks and renormalised.  Returns 0. */
int oracle_route_topk(const float* logits, int64_t T, int32_t E, int32_t k,
                      int32_t* topk_idx, float* topk_w) {
    unsigned char* taken = (unsigned char*)malloc(E > 0 ? (size_t)E : 1u);
    double* z = (double*)malloc(sizeof(double) * (k > 0 ? (size_t)k : 1u));
    for (int64_t t = 0; t < T; ++t) {
        const float* L = logits + t * E;
        memset(taken, 0, (size_t)E);
        for (int32_t j = 0; j < k; ++j) {          /* k rounds of argmax */
            int32_t best = -1;
            for (int32_t e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || L[e] > L[best]) best = e;  /* ties keep lower id */
            }
            taken[best] = 1;
            topk_idx[t * k + j] = best;
        }
        double m = (double)L[topk_idx[t * k]];
        double sum = 0.0;
        for (int32_t j = 0; j < k; ++j) {
            z[j] = exp((double)L[topk_idx[t * k + j]] - m);
            sum += z[j];
        }
        for (int32_t j = 0; j < k; ++j) topk_w[t * k + j] = (float)(z[j] / sum);
    }
    free(taken);
    free(z);
    return 0;
}

/* ------------------------------------------------------------------ */
/* S1' group-limited route: at most M expert groups per token           */
/* ------------------------------------------------------------------ */
/* "Expert Parallelism" (aiwiki), "Hiding the latency", topology-aware
 * routing: DeepSeek-V3's router sends each token to at most 4 nodes, which
 * bounds the inter-node fan-out.  The page does not say how the nodes are
 * chosen.  Reading: the E experts form G equal groups of E/G consecutive
 * experts (a node = a logical rank's block, "How the sizes combine"); a
 * group's score is its largest logit; each token keeps the M groups with
 * the largest scores (ties: lower group id) and picks its top k among their
 * experts with the ordinary rule (logit descending, expert id ascending);
 * the weights are the softmax over the k picks.  With M = G this is
 * oracle_route_topk.  Needs G | E and k <= M * E / G.  Returns 0, or -1 on
 * invalid sizes. */
int oracle_route_topk_grouped(const float* logits, int64_t T, int32_t E, int32_t k, int32_t G,
                              int32_t M, int32_t* topk_idx, float* topk_w) {
    if (G < 1 || E % G != 0 || M < 1 || M > G || k < 1 || k > M * (E / G)) return -1;
    const int32_t per = E / G;
    float* score = (float*)malloc(sizeof(float) * (size_t)G);
    unsigned char* keep = (unsigned char*)calloc((size_t)G, 1);
    unsigned char* taken = (unsigned char*)calloc((size_t)E > 0 ? (size_t)E : 1u, 1);
    double* z = (double*)malloc(sizeof(double) * (size_t)k);
    for (int64_t t = 0; t < T; ++t) {
        const float* L = logits + t * E;
        for (int32_t g = 0; g < G; ++g) {
            float m = L[g * per];
            for (int32_t e = g * per + 1; e < (g + 1) * per; ++e)
                if (L[e] > m) m = L[e];
            score[g] = m;
            keep[g] = 0;
        }
        for (int32_t r = 0; r < M; ++r) {     /* the M best groups */
            int32_t best = -1;
            for (int32_t g = 0; g < G; ++g) {
                if (keep[g]) continue;
                if (best < 0 || score[g] > score[best]) best = g;   /* ties keep lower id */
            }
            keep[best] = 1;
        }
        for (int32_t e = 0; e < E; ++e) taken[e] = 0;
        for (int32_t j = 0; j < k; ++j) {     /* top k inside the kept groups */
            int32_t best = -1;
            for (int32_t e = 0; e < E; ++e) {
                if (taken[e] || !keep[e / per]) continue;
                if (best < 0 || L[e] > L[best]) best = e;
            }
            taken[best] = 1;
            topk_idx[t * k + j] = best;
        }
        double m = (double)L[topk_idx[t * k]];
        double sum = 0.0;
        for (int32_t j = 0; j < k; ++j) {
            z[j] = exp((double)L[topk_idx[t * k + j]] - m);
            sum += z[j];
        }
        for (int32_t j = 0; j < k; ++j) topk_w[t * k + j] = (float)(z[j] / sum);
    }
    free(score);
    free(keep);
    free(taken);
    free(z);
    return 0;
}

/* ------------------------------------------------------------------ */
/* S2 dispatch layout: histogram, exclusive scan, stable counting sort */
/* ------------------------------------------------------------------ */
/* Pair p = t*k + j goes to expert idx[p].  Slots are expert-major, ties by
 * pair index (a stable sort by destination, as the aiwiki sketch's argsort
 * read as stable); logical rank r's slab starts at the offset of its first
 * expert r*E/W.  Pairs whose expert id is outside [0, E) are skipped:
 * slot_of_pair = -1, and slots past the last valid one hold -1.  Returns
 * the number of skipped pairs. */
int64_t oracle_dispatch_layout(const int32_t* idx, int64_t T, int32_t k, int32_t E,
                               int32_t W, int32_t* counts, int32_t* offsets,
                               int32_t* rank_offsets, int32_t* slot_of_pair,
                               int32_t* pair_of_slot) {
    int64_t N = T * k, bad = 0;
    for (int32_t e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t p = 0; p < N; ++p) {
        int32_t e = idx[p];
        if (e < 0 || e >= E) { ++bad; continue; }
        counts[e] += 1;
    }
    offsets[0] = 0;
    for (int32_t e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    for (int32_t r = 0; r <= W; ++r) rank_offsets[r] = offsets[(int64_t)r * E / W];
    int32_t* fill = (int32_t*)calloc(E > 0 ? (size_t)E : 1u, sizeof(int32_t));
    for (int64_t p = 0; p < N; ++p) {
        int32_t e = idx[p];
        if (e < 0 || e >= E) { slot_of_pair[p] = -1; continue; }
        int32_t s = offsets[e] + fill[e]++;
        slot_of_pair[p] = s;
        pair_of_slot[s] = (int32_t)p;
    }
    for (int64_t s = offsets[E]; s < N; ++s) pair_of_slot[s] = -1;
    free(fill);
    return bad;
}

/* ------------------------------------------------------------------ */
/* S2' fixed-capacity dispatch layout (token dropping)                  */
/* ------------------------------------------------------------------ */
/* "Expert Parallelism" (aiwiki), "Implementation", the closing note on
 * fixed capacity: with buffers of a fixed size every destination's size is
 * known in advance, and the tokens that do not fit are dropped.  Reading
 * (the page gives neither the size nor the drop rule): every expert e owns
 * a fixed slab of C rows, [e*C, (e+1)*C); its pairs, taken in pair order
 * (the stable order of the dropless layout), fill the slab from the top,
 * and the pairs past the C-th are dropped (slot_of_pair = -1), so the
 * earliest pairs keep their place.  counts[e] = min(#pairs of e, C) (the
 * rows the experts compute), offsets[e] = e*C, rank_offsets[r] =
 * offsets[r*E/W]; slab rows nobody fills hold pair_of_slot = -1.  Pairs
 * with an expert id outside [0, E) are skipped as in the dropless layout.
 * pair_of_slot has E*C entries.  Returns the number of dropped pairs;
 * *skipped receives the number of out-of-range ids. */
int64_t oracle_dispatch_layout_capacity(const int32_t* idx, int64_t T, int32_t k, int32_t E,
                                        int32_t W, int32_t C, int32_t* counts,
                                        int32_t* offsets, int32_t* rank_offsets,
                                        int32_t* slot_of_pair, int32_t* pair_of_slot,
                                        int64_t* skipped) {
    int64_t N = T * k, dropped = 0, bad = 0;
    for (int32_t e = 0; e < E; ++e) counts[e] = 0;
    for (int32_t e = 0; e <= E; ++e) offsets[e] = e * C;
    for (int32_t r = 0; r <= W; ++r) rank_offsets[r] = offsets[(int64_t)r * E / W];
    for (int64_t s = 0; s < (int64_t)E * C; ++s) pair_of_slot[s] = -1;
    for (int64_t p = 0; p < N; ++p) {
        int32_t e = idx[p];
        if (e < 0 || e >= E) { slot_of_pair[p] = -1; ++bad; continue; }
        if (counts[e] >= C) { slot_of_pair[p] = -1; ++dropped; continue; }
        int32_t s = offsets[e] + counts[e]++;
        slot_of_pair[p] = s;
        pair_of_slot[s] = (int32_t)p;
    }
    if (skipped) *skipped = bad;
    return dropped;
}

/* ------------------------------------------------------------------ */
/* S3 permute: xp[s] = x[pair_of_slot[s] / k], optional FP8 payload     */
/* ------------------------------------------------------------------ */
/* Same-dtype payload: a bitwise row copy.  FP8 payload: for every
 * 128-element block of the token's row, scale = amax / 448 (fp32 IEEE
 * division; 1 when amax is 0) and q = e4m3(x / scale) (fp32 IEEE division,
 * then round-to-nearest-even with saturation).  Slots holding -1 are not
 * written.  Returns 0, or -1 for an unsupported dtype pair. */
int oracle_permute(const void* x, int x_dt, int64_t T, int32_t H, int32_t k,
                   const int32_t* pair_of_slot, int64_t n_slots, void* xp, int xp_dt,
                   float* xp_scales) {
    (void)T;
    size_t eb = (x_dt == OR_F32) ? 4 : 2;
    if (xp_dt == x_dt) {
        for (int64_t s = 0; s < n_slots; ++s) {
            int32_t p = pair_of_slot[s];
            if (p < 0) continue;
            memcpy((char*)xp + (size_t)s * H * eb, (const char*)x + (size_t)(p / k) * H * eb,
                   (size_t)H * eb);
        }
        return 0;
    }
    if (xp_dt != OR_E4M3 || (H % 128) != 0) return -1;
    int32_t nb = H / 128;
    for (int64_t s = 0; s < n_slots; ++s) {
        int32_t p = pair_of_slot[s];
        if (p < 0) continue;
        int64_t t = p / k;
        for (int32_t b = 0; b < nb; ++b) {
            float amax = 0.0f;
            for (int32_t i = 0; i < 128; ++i) {
                float v = (float)load_elem(x, x_dt, t * H + b * 128 + i);
                if (fabsf(v) > amax) amax = fabsf(v);
            }
            float scale = amax / 448.0f;
            if (scale == 0.0f) scale = 1.0f;
            xp_scales[s * nb + b] = scale;
            for (int32_t i = 0; i < 128; ++i) {
                float v = (float)load_elem(x, x_dt, t * H + b * 128 + i);
                float r = v / scale;
                ((uint8_t*)xp)[s * H + b * 128 + i] = e4m3_from_float(r);
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* S4 grouped SwiGLU expert FFN                                        */
/* ------------------------------------------------------------------ */
/* For local expert j (global e = expert_begin + j) and every slot s in
 * [offsets[e], offsets[e+1]):
 *     g_i = sum_h A[s,h] W13[j, i, h],  u_i = sum_h A[s,h] W13[j, I+i, h]
 *     h_i = silu(g_i) * u_i,  silu(g) = g / (1 + exp(-g))
 *     y_o = sum_i h_i W2[j, o, i]
 * A is the payload row as a real number; for the FP8 payload it is the
 * bf16 rounding of the fp32 product decode(q) * scale.  The down
 * projection consumes h rounded to the weight dtype (as the path stores
 * it); h and y are written in out_dt (fp64 = unrounded, or a storage type).
 * row_mask (indexed by slot, may be NULL) restricts the work to a sample
 * of rows.  Returns the number of rows computed. */
int64_t oracle_grouped_gemm(const void* xp, int xp_dt, const float* xp_scales,
                            const int32_t* offsets, int32_t expert_begin,
                            int32_t n_experts, int32_t H, int32_t I, const void* w13,
                            const void* w2, int w_dt, const uint8_t* row_mask, void* h,
                            void* y, int out_dt) {
    int64_t s_lo = offsets[expert_begin], s_hi = offsets[expert_begin + n_experts];
    int64_t done = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : done)
    for (int64_t s = s_lo; s < s_hi; ++s) {
        if (row_mask && !row_mask[s]) continue;
        int32_t j = expert_begin;
        while (offsets[j + 1] <= s) ++j;          /* expert owning slot s */
        j -= expert_begin;
        double* a = (double*)malloc(sizeof(double) * (size_t)H);
        double* hv = (double*)malloc(sizeof(double) * (size_t)I);
        for (int32_t c = 0; c < H; ++c) {
            if (xp_dt == OR_E4M3) {
                float dq = (float)e4m3_to_double(((const uint8_t*)xp)[s * H + c]);
                float prod = dq * xp_scales[s * (H / 128) + c / 128];
                a[c] = bf16_to_double(bf16_from_double((double)prod));
            } else {
                a[c] = load_elem(xp, xp_dt, s * H + c);
            }
        }
        int64_t w13_base = (int64_t)j * 2 * I * H, w2_base = (int64_t)j * H * I;
        for (int32_t i = 0; i < I; ++i) {
            double g = 0.0, u = 0.0;
            for (int32_t c = 0; c < H; ++c) {
                g += a[c] * load_elem(w13, w_dt, w13_base + (int64_t)i * H + c);
                u += a[c] * load_elem(w13, w_dt, w13_base + (int64_t)(I + i) * H + c);
            }
            double v = g / (1.0 + exp(-g)) * u;
            store_elem(h, out_dt, s * I + i, v);
            hv[i] = round_to(w_dt, v);                 /* the down projection reads stored h */
        }
        for (int32_t o = 0; o < H; ++o) {
            double acc = 0.0;
            for (int32_t i = 0; i < I; ++i)
                acc += hv[i] * load_elem(w2, w_dt, w2_base + (int64_t)o * I + i);
            store_elem(y, out_dt, s * H + o, acc);
        }
        free(a);
        free(hv);
        done += 1;
    }
    return done;
}

/* ------------------------------------------------------------------ */
/* S5' FP8 combine payload: y as e4m3 codes with per-128 block scales   */
/* ------------------------------------------------------------------ */
/* "Expert parallelism and all-to-all", "Traffic math": the figure of
 * 2 * k * H * bytes per token assumes 1-byte activations both ways, i.e.
 * the experts' outputs also travel back as FP8.  Reading: per 128-element
 * block of each y row's fp32 values, scale = amax / 448 (fp32 IEEE
 * division; 1 when amax is 0) as for the dispatch payload, and q =
 * e4m3(y * r) with r = 1 / scale (one fp32 IEEE division per block, then an
 * fp32 product per element; round-to-nearest-even, saturating): the
 * combine payload has as many elements as the GEMM's outputs, so the
 * per-element IEEE division of the dispatch payload is replaced by a
 * product.  The combine uses decode(q) * scale as an fp32 product.
 * oracle_quantize_rows_e4m3 quantises rows of fp32 values; the caller
 * passes fp32(y). */
int oracle_quantize_rows_e4m3(const float* v, int64_t rows, int32_t H, uint8_t* q,
                              float* scales) {
    if ((H % 128) != 0) return -1;
    const int32_t nb = H / 128;
    for (int64_t r = 0; r < rows; ++r) {
        for (int32_t b = 0; b < nb; ++b) {
            const float* blk = v + r * H + b * 128;
            float amax = 0.0f;
            for (int32_t i = 0; i < 128; ++i)
                if (fabsf(blk[i]) > amax) amax = fabsf(blk[i]);
            float scale = amax / 448.0f;
            if (scale == 0.0f) scale = 1.0f;
            scales[r * nb + b] = scale;
            const float rs = 1.0f / scale;
            for (int32_t i = 0; i < 128; ++i) q[r * H + b * 128 + i] = e4m3_from_float(blk[i] * rs);
        }
    }
    return 0;
}

/* Combine from an FP8 y: out[t] = sum_j w[t,j] * (float)(decode(q) * scale)
 * for each kept pick, summed in fp64 in j order (out_dt fp64: unrounded). */
int oracle_combine_e4m3(const uint8_t* q, const float* scales, const int32_t* slot_of_pair,
                        const float* topk_w, int64_t T, int32_t k, int32_t H, void* out,
                        int out_dt) {
    if ((H % 128) != 0) return -1;
    const int32_t nb = H / 128;
    double* acc = (double*)malloc(sizeof(double) * (size_t)H);
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t c = 0; c < H; ++c) acc[c] = 0.0;
        for (int32_t j = 0; j < k; ++j) {
            const int32_t s = slot_of_pair[t * k + j];
            if (s < 0) continue;
            const double w = (double)topk_w[t * k + j];
            for (int32_t c = 0; c < H; ++c) {
                const float yv = (float)(e4m3_to_double(q[(int64_t)s * H + c]) *
                                         (double)scales[(int64_t)s * nb + c / 128]);
                acc[c] += w * (double)yv;
            }
        }
        for (int32_t c = 0; c < H; ++c) store_elem(out, out_dt, t * H + c, acc[c]);
    }
    free(acc);
    return 0;
}

/* ------------------------------------------------------------------ */
/* S5 combine: out[t] = sum_j w[t,j] * y[slot_of_pair[t*k+j]]          */
/* ------------------------------------------------------------------ */
/* The un-permute of the aiwiki sketch (y[order] = back) fused with the
 * router-weighted sum into the token's home row, in fp64; out_dt fp64
 * returns it unrounded.  Skipped pairs (slot -1) add nothing.  Returns 0. */
int oracle_combine(const void* y, int y_dt, const int32_t* slot_of_pair,
                   const float* topk_w, int64_t T, int32_t k, int32_t H, void* out,
                   int out_dt) {
    double* acc = (double*)malloc(sizeof(double) * (size_t)H);
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t c = 0; c < H; ++c) acc[c] = 0.0;
        for (int32_t j = 0; j < k; ++j) {
            int32_t s = slot_of_pair[t * k + j];
            if (s < 0) continue;
            double w = (double)topk_w[t * k + j];
            for (int32_t c = 0; c < H; ++c) acc[c] += w * load_elem(y, y_dt, (int64_t)s * H + c);
        }
        for (int32_t c = 0; c < H; ++c) store_elem(out, out_dt, t * H + c, acc[c]);
    }
    free(acc);
    return 0;
}

/* ------------------------------------------------------------------ */
/* The all_reduce form of the layer: per-rank partial sums, then their  */
/* sum over ranks                                                      */
/* ------------------------------------------------------------------ */
/* Transformers docs, "Expert parallelism", "Choosing an implementation",
 * the all_reduce row: no token moves; every rank runs its own experts over
 * the whole batch it shares with the other ranks, and the ranks' outputs
 * are summed by an all-reduce.  Rank r's experts own the slots
 * [rank_offsets[r], rank_offsets[r+1]) of the layout, so its contribution
 * to token t is
 *     partial_r[t] = sum over j with slot_of_pair[t*k+j] in that range of
 *                    topk_w[t,j] * y[slot_of_pair[t*k+j]],
 * zero for a token none of whose picks it owns.  fp64; out_dt fp64 returns
 * it unrounded.  Returns 0, or -1 if rank is outside [0, world). */
int oracle_combine_rank(const void* y, int y_dt, const int32_t* slot_of_pair,
                        const float* topk_w, int64_t T, int32_t k, int32_t H,
                        const int32_t* rank_offsets, int32_t world, int32_t rank, void* out,
                        int out_dt) {
    if (rank < 0 || rank >= world) return -1;
    const int32_t lo = rank_offsets[rank], hi = rank_offsets[rank + 1];
    double* acc = (double*)malloc(sizeof(double) * (size_t)H);
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t c = 0; c < H; ++c) acc[c] = 0.0;
        for (int32_t j = 0; j < k; ++j) {
            const int32_t s = slot_of_pair[t * k + j];
            if (s < lo || s >= hi) continue;   /* another rank's pick, or dropped (-1) */
            const double w = (double)topk_w[t * k + j];
            for (int32_t c = 0; c < H; ++c) acc[c] += w * load_elem(y, y_dt, (int64_t)s * H + c);
        }
        for (int32_t c = 0; c < H; ++c) store_elem(out, out_dt, t * H + c, acc[c]);
    }
    free(acc);
    return 0;
}

/* The all-reduce's sum: out[i] = partials[0][i] + ... + partials[n-1][i],
 * each partial read in its own dtype, summed in fp64 and rounded once to
 * out_dt.  n_elems elements per partial.  Returns 0. */
int oracle_reduce_partials(const void* partials, int p_dt, int32_t n, int64_t n_elems,
                           void* out, int out_dt) {
    for (int64_t i = 0; i < n_elems; ++i) {
        double acc = 0.0;
        for (int32_t r = 0; r < n; ++r) acc += load_elem(partials, p_dt, (int64_t)r * n_elems + i);
        store_elem(out, out_dt, i, acc);
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Expert parallelism over W ranks: the dispatch plan                   */
/* ------------------------------------------------------------------ */
/* "Expert Parallelism" (aiwiki), "The two all-to-alls" and
 * "Implementation": every rank sends each routed row to the owner of its
 * expert, and a count exchange first tells every owner how many rows will
 * arrive from each peer.  Rank r owns experts [r*Er, (r+1)*Er), Er = E/W
 * ("Expert parallelism" (Transformers), "How the sizes combine").
 *
 * counts_all[s*E + e] is the number of rows rank s routes to expert e (its
 * own layout's expert_counts, after the count exchange).  Reading of the
 * receive order (the pages' all_to_all_single delivers one chunk per source
 * rank; here the chunks are laid out so that each local expert's rows are
 * one contiguous segment): an owner's receive buffer holds its experts one
 * after the other; inside an expert, the rows of rank 0 come first, then
 * rank 1's, and so on, each source's rows in its own slot order.  For
 * rank `rank` this writes
 *   send_base[e]      (e = 0..E-1) the row of owner(e)'s receive buffer at
 *                     which rank's rows for expert e begin;
 *   recv_offsets[j]   (j = 0..Er) the row at which local expert j begins
 *                     in rank's own receive buffer (recv_offsets[Er] = the
 *                     rows it receives),
 * and returns the rows rank receives, or -1 for W not dividing E or a rank
 * outside [0, W). */
int64_t oracle_ep_plan(const int32_t* counts_all, int32_t W, int32_t E, int32_t rank,
                       int32_t* send_base, int32_t* recv_offsets) {
    if (W < 1 || E < 1 || E % W != 0 || rank < 0 || rank >= W) return -1;
    int32_t Er = E / W;
    int64_t mine = 0;
    for (int32_t r = 0; r < W; ++r) {
        int64_t row = 0;   /* rows of owner r's buffer filled so far */
        for (int32_t j = 0; j < Er; ++j) {
            int32_t e = r * Er + j;
            int64_t before = 0, all = 0;
            for (int32_t s = 0; s < W; ++s) {
                if (s < rank) before += counts_all[(int64_t)s * E + e];
                all += counts_all[(int64_t)s * E + e];
            }
            send_base[e] = (int32_t)(row + before);
            if (r == rank) recv_offsets[j] = (int32_t)row;
            row += all;
        }
        if (r == rank) {
            recv_offsets[Er] = (int32_t)row;
            mine = row;
        }
    }
    return mine;
}
