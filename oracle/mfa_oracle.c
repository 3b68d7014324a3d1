/*
 * mfa_oracle.c -- plain, slow, float64 CPU oracle for MFA decode attention and
 * the MFA low-rank query projection.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or load
 * this file: only the tests, the smoke check and the benchmark's CPU-baseline
 * leg use it. It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (Step-3 page, "Key points -> Architecture"): every decode
 * token has 64 query heads of dimension 256 that all attend over ONE shared key
 * head and ONE shared value head of dimension 256; the queries come out of a
 * 2048-wide low-rank bottleneck fed by the 7168-wide hidden state. The pages
 * print no attention formula; the plain reading used here is scaled dot-product
 * attention with a softmax over the cached tokens:
 *
 *     s[t]      = scale * sum_i q[b,h,i] * K_b[t,i]           (t < L_b)
 *     w[t]      = exp(s[t] - max_u s[u]) / sum_u exp(s[u] - max_u s[u])
 *     out[b,h,:] = sum_t w[t] * V_b[t,:]
 *     lse[b,h]   = max_u s[u] + log(sum_u exp(s[u] - max_u s[u]))
 *
 * K_b / V_b are either a contiguous per-sequence slab or are gathered through a
 * page table (PagedAttention, cited in the Step-3 page's reference list): token
 * t of sequence b lives in physical page page_table[b][t / page_size], row
 * t % page_size. FP8 caches hold E4M3 codes (the pages deploy attention in FP8);
 * the dequantised value is decode_e4m3(code) * k_scale (resp. v_scale).
 * An empty sequence (L_b = 0) has no softmax; this oracle defines its output as
 * zeros and its lse as -inf.
 *
 * The projection (same page, "Queries pass through a 2048-dim low-rank
 * bottleneck") is q = (x * W_qa) * W_qb with no bias, norm or activation, all in
 * float64 from the bf16 inputs.
 *
 * The key/value append (below) projects the new token's hidden state into the
 * shared K and V heads and stores the rounded rows into the cache.
 *
 * Every input arrives as the exact bit pattern the GPU sees (bf16 bits or E4M3
 * codes) and is up-converted exactly to double here; all arithmetic is double.
 *
 * Build: gcc -O2 -fno-fast-math -fopenmp -shared -fPIC mfa_oracle.c -lm
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stdlib.h>

#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_BF16 = 0, OR_F32 = 1, OR_E4M3 = 2 };

/* bf16 is the top half of an IEEE binary32: shift into place, reinterpret. */
static double bf16_bits_to_double(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* OCP FP8 E4M3 ("e4m3fn"): 1 sign bit, 4 exponent bits (bias 7), 3 mantissa
 * bits, no infinities; S.1111.111 is NaN. Exponent field 0 is subnormal:
 * 2^-6 * m/8. Otherwise 2^(e-7) * (1 + m/8). */
double mfa_oracle_e4m3_to_double(uint8_t code) {
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double mag;
    if (e == 0xF && m == 0x7) return NAN;
    if (e == 0)
        mag = ldexp((double)m / 8.0, -6);
    else
        mag = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -mag : mag;
}

/* One cached element as a double (before any per-tensor scale). */
static double cache_elem(const void* base, int dtype, int64_t idx) {
    if (dtype == OR_E4M3) return mfa_oracle_e4m3_to_double(((const uint8_t*)base)[idx]);
    if (dtype == OR_F32) return (double)((const float*)base)[idx];
    return bf16_bits_to_double(((const uint16_t*)base)[idx]);
}

/* Element index of K_b[t][i] (same for V): contiguous [B][Lmax][D] addressed by
 * strides, or paged [num_pages][page_size][D] through the page table. Returns -1
 * on an out-of-range page id. */
static int64_t cache_index(int b, int t, int i, int D, int64_t batch_stride, int64_t token_stride,
                           const int32_t* page_table, int max_pages, int page_size, int num_pages) {
    if (!page_table) return (int64_t)b * batch_stride + (int64_t)t * token_stride + i;
    int logical_page = t / page_size;
    int32_t phys = page_table[(int64_t)b * max_pages + logical_page];
    if (phys < 0 || phys >= num_pages) return -1;
    return ((int64_t)phys * page_size + (t % page_size)) * D + i;
}

/*
 * Decode attention for the (b, h) pairs listed in sel_b/sel_h (nsel of them), or
 * for all B*H pairs when sel_b == NULL (then out is [B][H][D], lse is [B][H]).
 * With a selection, out is [nsel][D] and lse is [nsel].
 *
 * q: [B][H][D] bf16 bits. k, v: cache of kv_dtype (0 bf16, 1 f32, 2 e4m3).
 * Contiguous caches (page_table == NULL) are addressed as b*batch_stride +
 * t*token_stride + i (element units). seq_lens[b] tokens of sequence b are used.
 * Returns 0, or -1 on an out-of-range page id / bad argument.
 */
int mfa_oracle_decode(int B, int H, int D, const uint16_t* q,
                      const void* k, const void* v, int kv_dtype,
                      int64_t batch_stride, int64_t token_stride,
                      const int32_t* page_table, int max_pages, int page_size, int num_pages,
                      const int32_t* seq_lens, double scale, double k_scale, double v_scale,
                      const int32_t* sel_b, const int32_t* sel_h, int nsel,
                      double* out, double* lse) {
    int npairs = sel_b ? nsel : B * H;
    int bad = 0;
    if (B < 0 || H <= 0 || D <= 0 || npairs < 0) return -1;

#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int p = 0; p < npairs; ++p) {
        int b = sel_b ? sel_b[p] : p / H;
        int h = sel_b ? sel_h[p] : p % H;
        double* o = out + (int64_t)p * D;
        int L = seq_lens[b];
        if (L <= 0) {
            for (int i = 0; i < D; ++i) o[i] = 0.0;
            if (lse) lse[p] = -INFINITY;
            continue;
        }
        double* s = (double*)malloc(sizeof(double) * (size_t)L);
        double* qv = (double*)malloc(sizeof(double) * (size_t)D);
        for (int i = 0; i < D; ++i) qv[i] = bf16_bits_to_double(q[((int64_t)b * H + h) * D + i]);

        /* scores */
        double smax = -INFINITY;
        for (int t = 0; t < L; ++t) {
            double acc = 0.0;
            for (int i = 0; i < D; ++i) {
                int64_t idx = cache_index(b, t, i, D, batch_stride, token_stride, page_table,
                                          max_pages, page_size, num_pages);
                if (idx < 0) { bad = 1; acc = 0.0; break; }
                acc += qv[i] * (cache_elem(k, kv_dtype, idx) * k_scale);
            }
            s[t] = scale * acc;
            if (s[t] > smax) smax = s[t];
        }
        /* softmax denominator */
        double denom = 0.0;
        for (int t = 0; t < L; ++t) denom += exp(s[t] - smax);
        /* weighted sum of value rows */
        for (int i = 0; i < D; ++i) o[i] = 0.0;
        for (int t = 0; t < L; ++t) {
            double w = exp(s[t] - smax) / denom;
            for (int i = 0; i < D; ++i) {
                int64_t idx = cache_index(b, t, i, D, batch_stride, token_stride, page_table,
                                          max_pages, page_size, num_pages);
                if (idx < 0) { bad = 1; break; }
                o[i] += w * (cache_elem(v, kv_dtype, idx) * v_scale);
            }
        }
        if (lse) lse[p] = smax + log(denom);
        free(s);
        free(qv);
    }
    return bad ? -1 : 0;
}

/*
 * Grouped-query attention (GQA; Ainslie et al., cited in the pages' reference
 * lists; the Step-3 summary page, "Key points -> Ablations", compares MFA with
 * it): H query heads of dimension D in G groups of H / G consecutive heads;
 * group g has its own key head and value head of dimension D, so a cached token
 * holds G key rows and G value rows. Head h belongs to group g = h / (H / G):
 *
 *     s[t]      = scale * sum_i q[b,h,i] * K_b[t,g,i]                 (t < L_b)
 *     out[b,h,:] = sum_t softmax(s)[t] * V_b[t,g,:],   lse as for MFA above
 *
 * q: [B][H][D] bf16 bits. k, v: bf16 bits, contiguous [B][Lmax][G][D] (strides
 * batch_stride, token_stride in elements; a token's G rows adjacent) or paged
 * [num_pages][page_size][G][D] through the page table. out [B][H][D], lse
 * [B][H]. Empty sequences: zeros, -inf. Returns 0, or -1 on an out-of-range page
 * id / bad argument.
 */
int mfa_oracle_gqa_decode(int B, int H, int G, int D, const uint16_t* q, const uint16_t* k,
                          const uint16_t* v, int64_t batch_stride, int64_t token_stride,
                          const int32_t* page_table, int max_pages, int page_size, int num_pages,
                          const int32_t* seq_lens, double scale, double* out, double* lse) {
    int bad = 0;
    if (B < 0 || H <= 0 || G <= 0 || D <= 0 || H % G != 0) return -1;
    const int heads_per_group = H / G;

#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int p = 0; p < B * H; ++p) {
        int b = p / H, h = p % H;
        int g = h / heads_per_group;
        double* o = out + (int64_t)p * D;
        int L = seq_lens[b];
        if (L <= 0) {
            for (int i = 0; i < D; ++i) o[i] = 0.0;
            lse[p] = -INFINITY;
            continue;
        }
        double* s = (double*)malloc(sizeof(double) * (size_t)L);
        int64_t* row = (int64_t*)malloc(sizeof(int64_t) * (size_t)L);
        /* element index of K_b[t][g][0] (same for V) */
        for (int t = 0; t < L; ++t) {
            if (page_table) {
                int32_t phys = page_table[(int64_t)b * max_pages + t / page_size];
                if (phys < 0 || phys >= num_pages) { bad = 1; row[t] = -1; continue; }
                row[t] = (((int64_t)phys * page_size + t % page_size) * G + g) * D;
            } else {
                row[t] = (int64_t)b * batch_stride + (int64_t)t * token_stride + (int64_t)g * D;
            }
        }
        double smax = -INFINITY;
        for (int t = 0; t < L; ++t) {
            double acc = 0.0;
            if (row[t] >= 0)
                for (int i = 0; i < D; ++i)
                    acc += bf16_bits_to_double(q[((int64_t)b * H + h) * D + i]) *
                           bf16_bits_to_double(k[row[t] + i]);
            s[t] = scale * acc;
            if (s[t] > smax) smax = s[t];
        }
        double denom = 0.0;
        for (int t = 0; t < L; ++t) denom += exp(s[t] - smax);
        for (int i = 0; i < D; ++i) o[i] = 0.0;
        for (int t = 0; t < L; ++t) {
            double w = exp(s[t] - smax) / denom;
            if (row[t] >= 0)
                for (int i = 0; i < D; ++i) o[i] += w * bf16_bits_to_double(v[row[t] + i]);
        }
        lse[p] = smax + log(denom);
        free(s);
        free(row);
    }
    return bad ? -1 : 0;
}

/*
 * Split-KV merge (Flash-Decoding, cited on the DeepSeek-V4 page): n partial
 * results of the same softmax over disjoint token ranges, each normalised within
 * its own range and carrying its range's log-sum-exp, merge into the result over
 * the union:
 *     lse* = max_s lse_s,  w_s = exp(lse_s - lse*),
 *     out  = sum_s w_s * out_s / sum_s w_s,   lse = lse* + log(sum_s w_s).
 * parts: [n][D], part_lse: [n]. Ranges whose lse is -inf (empty) carry no weight.
 */
void mfa_oracle_combine(int n, int D, const double* parts, const double* part_lse,
                        double* out, double* lse_out) {
    double m = -INFINITY;
    for (int s = 0; s < n; ++s)
        if (part_lse[s] > m) m = part_lse[s];
    for (int i = 0; i < D; ++i) out[i] = 0.0;
    if (m == -INFINITY) {
        if (lse_out) *lse_out = -INFINITY;
        return;
    }
    double wsum = 0.0;
    for (int s = 0; s < n; ++s) {
        double w = exp(part_lse[s] - m);
        wsum += w;
        for (int i = 0; i < D; ++i) out[i] += w * parts[(int64_t)s * D + i];
    }
    for (int i = 0; i < D; ++i) out[i] /= wsum;
    if (lse_out) *lse_out = m + log(wsum);
}

/*
 * Low-rank query projection: c = x * W_qa ([B][Dm] x [Dm][R]), q = c * W_qb
 * ([B][R] x [R][N]); all row-major bf16 bits, result q in double [B][N].
 * The latent c is kept in double (no rounding).
 */
void mfa_oracle_query_proj(int B, int Dm, int R, int N, const uint16_t* x,
                           const uint16_t* w_qa, const uint16_t* w_qb, double* q_out) {
    double* c = (double*)calloc((size_t)B * R, sizeof(double));
#pragma omp parallel for schedule(static)
    for (int r = 0; r < R; ++r) {
        for (int b = 0; b < B; ++b) {
            double acc = 0.0;
            for (int k = 0; k < Dm; ++k)
                acc += bf16_bits_to_double(x[(int64_t)b * Dm + k]) *
                       bf16_bits_to_double(w_qa[(int64_t)k * R + r]);
            c[(int64_t)b * R + r] = acc;
        }
    }
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n) {
        for (int b = 0; b < B; ++b) {
            double acc = 0.0;
            for (int r = 0; r < R; ++r)
                acc += c[(int64_t)b * R + r] * bf16_bits_to_double(w_qb[(int64_t)r * N + n]);
            q_out[(int64_t)b * N + n] = acc;
        }
    }
    free(c);
}

/*
 * New-token key/value projection and cache append. The pages print no W_k or
 * W_v; the plain reading of "one shared key head and one shared value head of
 * dimension 256" fed by the 7168-wide hidden state is k = x * W_k and
 * v = x * W_v ([B][Dm] x [Dm][D], no bias), in double from the bf16 inputs.
 */
void mfa_oracle_kv_project(int B, int Dm, int D, const uint16_t* x, const uint16_t* w_k,
                           const uint16_t* w_v, double* k_out, double* v_out) {
#pragma omp parallel for schedule(static)
    for (int i = 0; i < D; ++i) {
        for (int b = 0; b < B; ++b) {
            double ak = 0.0, av = 0.0;
            for (int k = 0; k < Dm; ++k) {
                const double xv = bf16_bits_to_double(x[(int64_t)b * Dm + k]);
                ak += xv * bf16_bits_to_double(w_k[(int64_t)k * D + i]);
                av += xv * bf16_bits_to_double(w_v[(int64_t)k * D + i]);
            }
            k_out[(int64_t)b * D + i] = ak;
            v_out[(int64_t)b * D + i] = av;
        }
    }
}

/* The bf16 nearest to v (ties to even), as bits: 8 significant bits, exponent
 * range of binary32 (subnormals below 2^-126; beyond the largest finite value
 * the result is infinity). */
uint16_t mfa_oracle_bf16_round(double v) {
    if (isnan(v)) return 0x7FC0;
    const uint16_t sign = signbit(v) ? 0x8000 : 0;
    const double a = fabs(v);
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e);     /* a = f * 2^e, f in [0.5, 1): the leading bit has weight 2^(e-1) */
    int lead = e - 1;
    if (lead < -126) lead = -126; /* subnormal range: fixed quantum 2^-133 */
    double r = nearbyint(ldexp(a, 7 - lead)); /* significand in units of the last bit, ties to even */
    double q = ldexp(r, lead - 7);            /* the rounded magnitude */
    if (q >= ldexp(1.0, 128)) return sign | 0x7F80;
    float f = (float)q; /* exact: q has at most 8 significant bits in binary32's range */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | (u >> 16));
}

/* The E4M3 code nearest to v (ties to the code with an even mantissa),
 * saturating to +-448 beyond it; NaN to 0x7F. Searches all finite codes. */
uint8_t mfa_oracle_e4m3_encode(double v) {
    if (isnan(v)) return 0x7F;
    const uint8_t sign = signbit(v) ? 0x80 : 0;
    const double a = fabs(v);
    int best = 0;
    double best_d = INFINITY;
    for (int code = 0; code <= 0x7E; ++code) {
        const double d = fabs(mfa_oracle_e4m3_to_double((uint8_t)code) - a);
        if (d < best_d || (d == best_d && (code & 1) == 0)) {
            best_d = d;
            best = code;
        }
    }
    return (uint8_t)(sign | best);
}

/*
 * Output projection: the attention outputs of a token, its 64 heads x 256
 * concatenated (16384 values), times W_o back to the 7168-wide hidden state:
 * y = o * W_o ([B][K] x [K][N], no bias), in double from the bf16 inputs. The
 * pages name no W_o; this is the plain reading of an attention layer's output
 * projection to the hidden size.
 */
void mfa_oracle_out_proj(int B, int K, int N, const uint16_t* o, const uint16_t* w_o,
                         double* y_out) {
    /* every y[b][n] sums its K products in ascending k; W_o is walked row by row */
#pragma omp parallel for schedule(static)
    for (int b = 0; b < B; ++b) {
        double* y = y_out + (int64_t)b * N;
        for (int n = 0; n < N; ++n) y[n] = 0.0;
        for (int k = 0; k < K; ++k) {
            const double ov = bf16_bits_to_double(o[(int64_t)b * K + k]);
            const uint16_t* w = w_o + (int64_t)k * N;
            for (int n = 0; n < N; ++n) y[n] += ov * bf16_bits_to_double(w[n]);
        }
    }
}

/* Number of OpenMP threads a parallel region here would use (1 without OpenMP). */
int mfa_oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
