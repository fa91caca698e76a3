/*
 * oracle.c -- plain fp64 CPU oracle for paged FP8-KV decode attention.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline / reference arm may load this file's library.
 * The product path (the CUDA library) never calls it and shares no code,
 * header, table or constant with it.
 *
 * Sources, cited by page title and section:
 *   [T]  "大模型推理优化：量化、压缩与安全验证" (Chinese translation of the
 *        first-party post), sections "量化 KV cache" and "保护共享 KV cache".
 *   [S]  siami.tw editorial on Cloudflare's Kimi/GLM inference, section
 *        "KV 快取量化" (Table 1) and "共享 KV 快取的完整性檢查" (Table 3).
 *   [R]  remio.ai commentary "Cloudflare 小型模型服务降低内存占用，但安全性成为考验",
 *        section "共享 KV 缓存安全性成为生产问题".
 *   [OCP] OCP 8-bit Floating Point Specification (OFP8), E4M3 encoding, as
 *        published with Micikevicius et al., "FP8 Formats for Deep Learning"
 *        (2022): 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits,
 *        no infinities, S.1111.111 is NaN, largest finite value 448.
 *
 * Everything here is written for a reader to check by eye: no blocking, no
 * fusion, no reordering beyond the definitions.  Floating point is fp64
 * except where the method itself fixes fp32 (the quantiser's division).
 *
 * Readings of points the pages leave open (each is also listed in the
 * design notes of the repository):
 *   - Scale granularity: one fp32 scale for K and one for V (per tensor).
 *   - Quantise: y = fp32(x) / fp32(scale) as one correctly rounded fp32
 *     division, then round y to E4M3 with round-to-nearest-even; any |y|
 *     above 448 saturates to +-448 (Inf included); a NaN input x becomes
 *     S.1111.111 with the sign bit of x (the sign of a NaN quotient is not
 *     fixed by IEEE 754); a zero keeps its sign.
 *   - Dequantise: x = decode(code) * scale, in fp64.
 *   - Attention: s_t = sm_scale * q . k_t over t < L (L counts the new
 *     token), LSE = m + ln(sum exp(s_t - m)), o = sum exp(s_t - LSE) v_t.
 *   - A request that is aborted, whose length is outside [1, MP*P], or whose
 *     page table names a page outside [0, NP) gets o = 0 and LSE = -inf.
 *   - Tag check: only the ceil(L/P) used entries are compared; an entry
 *     naming a page outside [0, NP) counts as a mismatch; a length outside
 *     [1, MP*P] fails the check as a whole.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* bf16 and E4M3 codecs                                                     */
/* ------------------------------------------------------------------------ */

/* bf16 is the upper half of an IEEE binary32 word. */
double orc_bf16_to_double(uint16_t bits)
{
    uint32_t w = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return (double)f;
}

/* Round an fp64 value to the nearest bf16 (8 significant bits, binary32
 * exponent range), ties to even; results beyond the largest finite bf16
 * become infinities, as IEEE round-to-nearest prescribes. */
uint16_t orc_bf16_from_double(double x)
{
    if (isnan(x))
        return signbit(x) ? 0xFFC0u : 0x7FC0u;
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    double a = fabs(x);
    if (a == 0.0)
        return sign;
    if (isinf(a))
        return sign | 0x7F80u;
    int e;
    frexp(a, &e);                 /* a = f * 2^e with f in [0.5, 1) */
    int unit_exp = (e - 1) - 7;   /* weight of the last kept bit    */
    if (unit_exp < -133)          /* subnormal range: fixed quantum */
        unit_exp = -133;
    double n = nearbyint(ldexp(a, -unit_exp)); /* exact scaling, RNE */
    double r = ldexp(n, unit_exp);
    if (r >= ldexp(1.0, 128))
        return sign | 0x7F80u;
    float rf = (float)r;          /* exact: r has at most 8 significant bits */
    uint32_t w;
    memcpy(&w, &rf, sizeof w);
    return sign | (uint16_t)((w >> 16) & 0x7FFFu);
}

/* [OCP] E4M3: value = (-1)^s * 2^(e-7) * (1 + m/8) for e in 1..15,
 * (-1)^s * 2^-6 * (m/8) for e = 0; S.1111.111 is NaN; no infinities. */
double orc_e4m3_decode(uint8_t c)
{
    int s = c >> 7;
    int e = (c >> 3) & 0xF;
    int m = c & 0x7;
    double v;
    if (e == 0xF && m == 0x7)
        return s ? -NAN : NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

/* Round a binary32 value to E4M3: nearest representable magnitude, ties to
 * the code whose last mantissa bit is 0, saturating at 448. */
uint8_t orc_e4m3_encode(float y)
{
    uint8_t sign = signbit(y) ? 0x80u : 0x00u;
    if (isnan(y))
        return sign | 0x7Fu;
    double a = fabs((double)y);
    if (a > 448.0)
        return sign | 0x7Eu;
    /* Non-negative finite codes 0x00..0x7E are increasing in value.  Find
     * the largest code whose value does not exceed a (binary search), then
     * pick between it and its successor. */
    int lo = 0, hi = 0x7E;
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if (orc_e4m3_decode((uint8_t)mid) <= a)
            lo = mid;
        else
            hi = mid - 1;
    }
    int k = lo;
    if (k < 0x7E) {
        double below = orc_e4m3_decode((uint8_t)k);
        double above = orc_e4m3_decode((uint8_t)(k + 1));
        double d_lo = a - below, d_hi = above - a;
        if (d_hi < d_lo || (d_hi == d_lo && ((k + 1) & 1) == 0))
            k = k + 1;
    }
    return sign | (uint8_t)k;
}

/* [T] "量化 KV cache": the cache is stored as FP8 e4m3.  The division is one
 * IEEE binary32 division (the file is built without contraction or fast
 * math, so this is exactly fp32 x / fp32 scale). */
uint8_t orc_quantize_bf16(uint16_t x_bits, float scale)
{
    uint32_t w = (uint32_t)x_bits << 16;
    float x;
    memcpy(&x, &w, sizeof x);
    /* IEEE 754 leaves the sign of a NaN produced by an operation unspecified,
     * so the NaN rule is stated on the input: a NaN x becomes S.1111.111 with
     * the sign bit of x. */
    if (isnan(x))
        return signbit(x) ? 0xFFu : 0x7Fu;
    volatile float y = x / scale;
    return orc_e4m3_encode(y);
}

/* Whole-array helpers so that the Python side can pin the codecs cheaply. */
void orc_e4m3_encode_array(const float* y, uint8_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = orc_e4m3_encode(y[i]);
}

void orc_quantize_bf16_array(const uint16_t* x, float scale, uint8_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = orc_quantize_bf16(x[i], scale);
}

void orc_bf16_from_double_array(const double* x, uint16_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = orc_bf16_from_double(x[i]);
}

/* ------------------------------------------------------------------------ */
/* Page-tag integrity check                                                 */
/* ------------------------------------------------------------------------ */

/* [T] "保护共享 KV cache", [S] "共享 KV 快取的完整性檢查", [R] "共享 KV 缓存安全性成为生产问题":
 * every physical page carries a tag that changes when the page is
 * reallocated; the server records, per request, the pages it expects and
 * their tags; before a supported decode op reads the cache the mapping is
 * checked and a request with any mismatch is aborted.
 *
 * abort[b] = 1 iff L_b is outside [1, MP*P], or some used entry
 * j < ceil(L_b/P) names a page outside [0, NP) or a page whose current tag
 * differs from expected_tags[b][j].  Returns the number of aborted requests. */
int32_t orc_kv_tag_check(const uint32_t* page_tags, int32_t num_pages,
                         const int32_t* page_table, const uint32_t* expected_tags,
                         int32_t max_pages, const int32_t* seq_lens, int32_t batch,
                         int32_t page_size, uint8_t* abort_out)
{
    int32_t aborted = 0;
    for (int32_t b = 0; b < batch; ++b) {
        int32_t L = seq_lens[b];
        int bad = 0;
        if (L < 1 || (int64_t)L > (int64_t)max_pages * page_size) {
            bad = 1;
        } else {
            int32_t used = (L + page_size - 1) / page_size;
            for (int32_t j = 0; j < used; ++j) {
                int32_t pid = page_table[(int64_t)b * max_pages + j];
                if (pid < 0 || pid >= num_pages) {
                    bad = 1;
                } else if (page_tags[pid] != expected_tags[(int64_t)b * max_pages + j]) {
                    bad = 1;
                }
            }
        }
        abort_out[b] = (uint8_t)bad;
        aborted += bad;
    }
    return aborted;
}

/* [T] "保护共享 KV cache" and [R] "共享 KV 缓存安全性成为生产问题": a page's tag
 * changes whenever the page is reallocated (like a generation counter).
 * Every listed page id inside [0, NP) has its tag increased by one, modulo
 * 2^32, once per occurrence in the list; other ids are ignored. */
void orc_kv_retag_pages(uint32_t* page_tags, int32_t num_pages, const int32_t* pages, int32_t n)
{
    for (int32_t i = 0; i < n; ++i) {
        int32_t p = pages[i];
        if (p >= 0 && p < num_pages)
            page_tags[p] = page_tags[p] + 1u;
    }
}

/* The server records, per request, the tags it expects for its pages: for
 * every used entry j < ceil(L_b / P) that names a page inside [0, NP),
 * expected_tags[b][j] = page_tags[page_table[b][j]].  Entries naming a page
 * outside the pool, entries past the used ones and requests whose length is
 * outside [1, MP*P] are left unchanged. */
void orc_kv_expected_tags(const uint32_t* page_tags, int32_t num_pages,
                          const int32_t* page_table, int32_t max_pages,
                          const int32_t* seq_lens, int32_t batch, int32_t page_size,
                          uint32_t* expected_tags)
{
    for (int32_t b = 0; b < batch; ++b) {
        int32_t L = seq_lens[b];
        if (L < 1 || (int64_t)L > (int64_t)max_pages * page_size)
            continue;
        int32_t used = (L + page_size - 1) / page_size;
        for (int32_t j = 0; j < used; ++j) {
            int32_t pid = page_table[(int64_t)b * max_pages + j];
            if (pid >= 0 && pid < num_pages)
                expected_tags[(int64_t)b * max_pages + j] = page_tags[pid];
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Quantise-and-append of the new token                                     */
/* ------------------------------------------------------------------------ */

/* Cache layout: [num_pages][num_kv_heads][page_size][head_dim].  The new
 * token of request b sits at position L_b - 1 (L_b counts it), i.e. in page
 * page_table[b][(L_b-1)/P], slot (L_b-1) % P.  Requests that are aborted,
 * have a length outside [1, MP*P], or name a page outside [0, NP) are
 * skipped. */
void orc_kv_append_fp8(const uint16_t* k_new, const uint16_t* v_new,
                       const int32_t* page_table, int32_t max_pages,
                       const int32_t* seq_lens, int32_t batch, int32_t num_kv_heads,
                       int32_t head_dim, int32_t page_size, float k_scale, float v_scale,
                       uint8_t* k_cache, uint8_t* v_cache, int32_t num_pages,
                       const uint8_t* abort)
{
    for (int32_t b = 0; b < batch; ++b) {
        if (abort && abort[b])
            continue;
        int32_t L = seq_lens[b];
        if (L < 1 || (int64_t)L > (int64_t)max_pages * page_size)
            continue;
        int32_t pos = L - 1;
        int32_t pid = page_table[(int64_t)b * max_pages + pos / page_size];
        if (pid < 0 || pid >= num_pages)
            continue;
        int32_t slot = pos % page_size;
        for (int32_t h = 0; h < num_kv_heads; ++h) {
            for (int32_t d = 0; d < head_dim; ++d) {
                int64_t src = ((int64_t)b * num_kv_heads + h) * head_dim + d;
                int64_t dst = (((int64_t)pid * num_kv_heads + h) * page_size + slot) * head_dim + d;
                k_cache[dst] = orc_quantize_bf16(k_new[src], k_scale);
                v_cache[dst] = orc_quantize_bf16(v_new[src], v_scale);
            }
        }
    }
}

/* Same write for a BF16 cache: the value is stored unchanged. */
void orc_kv_append_bf16(const uint16_t* k_new, const uint16_t* v_new,
                        const int32_t* page_table, int32_t max_pages,
                        const int32_t* seq_lens, int32_t batch, int32_t num_kv_heads,
                        int32_t head_dim, int32_t page_size,
                        uint16_t* k_cache, uint16_t* v_cache, int32_t num_pages,
                        const uint8_t* abort)
{
    for (int32_t b = 0; b < batch; ++b) {
        if (abort && abort[b])
            continue;
        int32_t L = seq_lens[b];
        if (L < 1 || (int64_t)L > (int64_t)max_pages * page_size)
            continue;
        int32_t pos = L - 1;
        int32_t pid = page_table[(int64_t)b * max_pages + pos / page_size];
        if (pid < 0 || pid >= num_pages)
            continue;
        int32_t slot = pos % page_size;
        for (int32_t h = 0; h < num_kv_heads; ++h) {
            for (int32_t d = 0; d < head_dim; ++d) {
                int64_t src = ((int64_t)b * num_kv_heads + h) * head_dim + d;
                int64_t dst = (((int64_t)pid * num_kv_heads + h) * page_size + slot) * head_dim + d;
                k_cache[dst] = k_new[src];
                v_cache[dst] = v_new[src];
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* BF16 page -> FP8 page handoff                                            */
/* ------------------------------------------------------------------------ */

/* [S] "KV 快取量化" and [T] "量化 KV cache": prefill keeps a BF16 cache and
 * decode an FP8 one.  Handing a page over re-quantises every element with
 * the same rule as the append.  Page src_pages[i] of the BF16 pool becomes
 * page dst_pages[i] of the FP8 pool; a pair naming an id outside its pool
 * is skipped. */
void orc_kv_requant_pages_fp8(const uint16_t* src_pool, int32_t src_num_pages,
                              const int32_t* src_pages, uint8_t* dst_pool,
                              int32_t dst_num_pages, const int32_t* dst_pages,
                              int32_t n, int32_t num_kv_heads, int32_t page_size,
                              int32_t head_dim, float scale)
{
    int64_t page_elems = (int64_t)num_kv_heads * page_size * head_dim;
    for (int32_t i = 0; i < n; ++i) {
        int32_t s = src_pages[i], d = dst_pages[i];
        if (s < 0 || s >= src_num_pages || d < 0 || d >= dst_num_pages)
            continue;
        for (int64_t e = 0; e < page_elems; ++e)
            dst_pool[(int64_t)d * page_elems + e] =
                orc_quantize_bf16(src_pool[(int64_t)s * page_elems + e], scale);
    }
}

/* ------------------------------------------------------------------------ */
/* Paged decode attention                                                   */
/* ------------------------------------------------------------------------ */

/* Element d of token t of KV head hk of request b, dequantised to fp64.
 * kv_dtype 0: FP8 E4M3 codes times the per-tensor scale ([T] "量化 KV cache":
 * the FP8 attention kernel converts on every read); kv_dtype 1: BF16. */
static double kv_element(int kv_dtype, const void* cache, double scale,
                         int32_t pid, int32_t num_kv_heads, int32_t hk,
                         int32_t page_size, int32_t slot, int32_t head_dim, int32_t d)
{
    int64_t idx = (((int64_t)pid * num_kv_heads + hk) * page_size + slot) * head_dim + d;
    if (kv_dtype == 0)
        return orc_e4m3_decode(((const uint8_t*)cache)[idx]) * scale;
    return orc_bf16_to_double(((const uint16_t*)cache)[idx]);
}

/* Decode attention of one new query token per request over its paged
 * cache.  q: [B][Hq][D] bf16; caches [NP][Hkv][P][D]; page_table [B][MP];
 * query head h reads KV head h / (Hq/Hkv).  Outputs are fp64: out [B][Hq][D]
 * and lse [B][Hq] (natural log of the softmax normaliser of the scaled
 * scores).  items lists the (b * Hkv + kv_head) pairs to compute; NULL
 * means all of them.  Entries of out/lse outside the listed items are left
 * untouched. */
void orc_paged_decode_attn(int32_t kv_dtype, const uint16_t* q,
                           const void* k_cache, const void* v_cache,
                           float k_scale, float v_scale,
                           const int32_t* page_table, int32_t max_pages,
                           const int32_t* seq_lens, int32_t batch,
                           int32_t num_q_heads, int32_t num_kv_heads,
                           int32_t head_dim, int32_t page_size, int32_t num_pages,
                           float sm_scale, const uint8_t* abort,
                           const int32_t* items, int32_t n_items,
                           double* out, double* lse)
{
    int32_t group = num_q_heads / num_kv_heads;
    int32_t total = items ? n_items : batch * num_kv_heads;
    for (int32_t it = 0; it < total; ++it) {
        int32_t item = items ? items[it] : it;
        int32_t b = item / num_kv_heads;
        int32_t hk = item % num_kv_heads;
        int32_t L = seq_lens[b];

        int dead = (abort && abort[b]);
        if (L < 1 || (int64_t)L > (int64_t)max_pages * page_size)
            dead = 1;
        if (!dead) {
            int32_t used = (L + page_size - 1) / page_size;
            for (int32_t j = 0; j < used; ++j) {
                int32_t pid = page_table[(int64_t)b * max_pages + j];
                if (pid < 0 || pid >= num_pages)
                    dead = 1;
            }
        }

        double* scores = dead ? NULL : (double*)malloc(sizeof(double) * (size_t)L);
        for (int32_t g = 0; g < group; ++g) {
            int32_t h = hk * group + g;
            double* o = out + ((int64_t)b * num_q_heads + h) * head_dim;
            if (dead) {
                for (int32_t d = 0; d < head_dim; ++d)
                    o[d] = 0.0;
                lse[(int64_t)b * num_q_heads + h] = -INFINITY;
                continue;
            }
            const uint16_t* qh = q + ((int64_t)b * num_q_heads + h) * head_dim;

            /* scores s_t = sm_scale * sum_d q[d] k_t[d], for t < L */
            for (int32_t t = 0; t < L; ++t) {
                int32_t pid = page_table[(int64_t)b * max_pages + t / page_size];
                double dot = 0.0;
                for (int32_t d = 0; d < head_dim; ++d)
                    dot += orc_bf16_to_double(qh[d]) *
                           kv_element(kv_dtype, k_cache, (double)k_scale, pid, num_kv_heads,
                                      hk, page_size, t % page_size, head_dim, d);
                scores[t] = (double)sm_scale * dot;
            }
            /* m = max_t s_t (a NaN score makes everything NaN) */
            double m = -INFINITY;
            for (int32_t t = 0; t < L; ++t) {
                if (isnan(scores[t]) || isnan(m))
                    m = NAN;
                else if (scores[t] > m)
                    m = scores[t];
            }
            /* LSE = m + ln sum_t exp(s_t - m) */
            double sum = 0.0;
            for (int32_t t = 0; t < L; ++t)
                sum += exp(scores[t] - m);
            double lse_v = m + log(sum);
            lse[(int64_t)b * num_q_heads + h] = lse_v;

            /* o = sum_t exp(s_t - LSE) v_t */
            for (int32_t d = 0; d < head_dim; ++d)
                o[d] = 0.0;
            for (int32_t t = 0; t < L; ++t) {
                int32_t pid = page_table[(int64_t)b * max_pages + t / page_size];
                double w = exp(scores[t] - lse_v);
                for (int32_t d = 0; d < head_dim; ++d)
                    o[d] += w * kv_element(kv_dtype, v_cache, (double)v_scale, pid,
                                           num_kv_heads, hk, page_size, t % page_size,
                                           head_dim, d);
            }
        }
        free(scores);
    }
}

/* ------------------------------------------------------------------------ */
/* Split-K pieces and their log-sum-exp merge                               */
/* ------------------------------------------------------------------------ */
/*
 * The decomposition the CUDA path uses (not on the pages, which give no
 * kernel design): attention over a token range [t0, t1) of one query head
 * gives a partial (m, l, o) with m = max_t s_t, l = sum_t exp(s_t - m) and
 * the unnormalised o = sum_t exp(s_t - m) v_t; partials of disjoint ranges
 * covering the sequence merge into the head's output and LSE:
 *   M = max_s m_s,  l = sum_s l_s exp(m_s - M),
 *   out = sum_s o_s exp(m_s - M) / l,  LSE = M + ln l.
 * An empty range is the partial (-inf, 0, 0); merging only empty partials
 * gives out = 0 and LSE = -inf.  The scores s_t are those of
 * orc_paged_decode_attn (the caller passes a live request).
 */
void orc_attn_partial(int32_t kv_dtype, const uint16_t* q, const void* k_cache,
                      const void* v_cache, float k_scale, float v_scale,
                      const int32_t* page_table, int32_t max_pages, int32_t num_q_heads,
                      int32_t num_kv_heads, int32_t head_dim, int32_t page_size,
                      float sm_scale, int32_t b, int32_t h, int32_t t0, int32_t t1,
                      double* m_out, double* l_out, double* o_out)
{
    int32_t hk = h / (num_q_heads / num_kv_heads);
    const uint16_t* qh = q + ((int64_t)b * num_q_heads + h) * head_dim;
    for (int32_t d = 0; d < head_dim; ++d)
        o_out[d] = 0.0;
    *m_out = -INFINITY;
    *l_out = 0.0;
    if (t1 <= t0)
        return;
    double* scores = (double*)malloc(sizeof(double) * (size_t)(t1 - t0));
    double m = -INFINITY;
    for (int32_t t = t0; t < t1; ++t) {
        int32_t pid = page_table[(int64_t)b * max_pages + t / page_size];
        double dot = 0.0;
        for (int32_t d = 0; d < head_dim; ++d)
            dot += orc_bf16_to_double(qh[d]) *
                   kv_element(kv_dtype, k_cache, (double)k_scale, pid, num_kv_heads, hk,
                              page_size, t % page_size, head_dim, d);
        scores[t - t0] = (double)sm_scale * dot;
        if (scores[t - t0] > m)
            m = scores[t - t0];
    }
    double l = 0.0;
    for (int32_t t = t0; t < t1; ++t) {
        int32_t pid = page_table[(int64_t)b * max_pages + t / page_size];
        double w = exp(scores[t - t0] - m);
        l += w;
        for (int32_t d = 0; d < head_dim; ++d)
            o_out[d] += w * kv_element(kv_dtype, v_cache, (double)v_scale, pid, num_kv_heads,
                                       hk, page_size, t % page_size, head_dim, d);
    }
    free(scores);
    *m_out = m;
    *l_out = l;
}

void orc_lse_merge(int32_t n, int32_t head_dim, const double* m, const double* l,
                   const double* o, double* out, double* lse)
{
    double M = -INFINITY;
    for (int32_t s = 0; s < n; ++s)
        if (m[s] > M)
            M = m[s];
    for (int32_t d = 0; d < head_dim; ++d)
        out[d] = 0.0;
    if (M == -INFINITY) {
        *lse = -INFINITY;
        return;
    }
    double lsum = 0.0;
    for (int32_t s = 0; s < n; ++s) {
        if (m[s] == -INFINITY)
            continue;
        double w = exp(m[s] - M);
        lsum += l[s] * w;
        for (int32_t d = 0; d < head_dim; ++d)
            out[d] += o[(int64_t)s * head_dim + d] * w;
    }
    for (int32_t d = 0; d < head_dim; ++d)
        out[d] /= lsum;
    *lse = M + log(lsum);
}

/* ------------------------------------------------------------------------ */
/* INT4 weight dequantisation GEMV (decode)                                 */
/* ------------------------------------------------------------------------ */
/*
 * [T] section "压缩模型权重", [S] section "模型權重壓縮：GLM 5.2 從 705 GB
 * 縮到 421 GB" (Table 2) and [R] section "GLM 权重压缩改变了阶段权衡": model
 * weights are stored as 4-bit integers, streamed from memory once per
 * generated token, and expanded back to floating point before they are
 * multiplied.  The pages fix no format; the reading used here:
 *   - a code is a signed 4-bit integer in two's complement, -8..7;
 *   - W (n rows = output features, k columns) is stored in tiles of 128 rows
 *     x 256 columns, 16384 bytes each; tile (r, t) covers rows 128r.. and
 *     columns 256t.. and starts at byte (r * (k/256) + t) * 16384; inside
 *     it, row j's 128 bytes start at (j mod 128) * 128 and hold 32
 *     little-endian 32-bit words; word w holds the 8 columns
 *     c = 256t + 8w .. c + 7: bits 4i..4i+3 hold column c + 2i and bits
 *     16+4i..16+4i+3 hold column c + 2i + 1 (i = 0..3), i.e. the even
 *     columns in the low half-word and the odd ones in the high half-word;
 *   - every run of `group` consecutive columns of a row shares one bf16
 *     scale; the scales of 128-row block r and group g are 128 consecutive
 *     values starting at element (r * (k/group) + g) * 128;
 *   - w[j][i] = code * scale (exact in fp64), and
 *     y[b][j] = bf16_rne( sum_i x[b][i] * w[j][i] ) with x in bf16.
 */

/* Code of column i of row j as a signed integer. */
int32_t orc_int4_code(const uint8_t* w_tiles, int32_t k, int32_t j, int32_t i)
{
    int64_t tile = (int64_t)(j / 128) * (k / 256) + i / 256;
    int64_t at = tile * 16384 + (int64_t)(j % 128) * 128 + (int64_t)((i % 256) / 8) * 4;
    uint32_t word = (uint32_t)w_tiles[at] | ((uint32_t)w_tiles[at + 1] << 8) |
                    ((uint32_t)w_tiles[at + 2] << 16) | ((uint32_t)w_tiles[at + 3] << 24);
    int32_t m = i % 8;
    int32_t bit = (m % 2 == 0) ? 4 * (m / 2) : 16 + 4 * (m / 2);
    int32_t nibble = (int32_t)((word >> bit) & 0x0Fu);
    return nibble >= 8 ? nibble - 16 : nibble;
}

/* Scale of column i of row j. */
double orc_int4_scale(const uint16_t* scales, int32_t k, int32_t group, int32_t j, int32_t i)
{
    int64_t at = ((int64_t)(j / 128) * (k / group) + i / group) * 128 + j % 128;
    return orc_bf16_to_double(scales[at]);
}

/* All codes of rows [0, n) as int8, row-major [n][k]. */
void orc_int4_unpack(const uint8_t* w_tiles, int32_t n, int32_t k, int8_t* codes)
{
    for (int32_t j = 0; j < n; ++j)
        for (int32_t i = 0; i < k; ++i)
            codes[(int64_t)j * k + i] = (int8_t)orc_int4_code(w_tiles, k, j, i);
}

/*
 * y = x W^T for the rows listed in rows[0..nrows) (all n rows in order when
 * rows is NULL).  y_exact [batch][nrows] receives the fp64 sums, y
 * [batch][nrows] their bf16 rounding; either may be NULL.
 */
void orc_int4_gemv(const uint16_t* x, const uint8_t* w_tiles, const uint16_t* scales,
                   int32_t batch, int32_t n, int32_t k, int32_t group,
                   const int32_t* rows, int32_t nrows, double* y_exact, uint16_t* y)
{
    if (rows == NULL)
        nrows = n;
    for (int32_t r = 0; r < nrows; ++r) {
        int32_t j = rows ? rows[r] : r;
        for (int32_t b = 0; b < batch; ++b) {
            double sum = 0.0;
            for (int32_t i = 0; i < k; ++i) {
                double w = (double)orc_int4_code(w_tiles, k, j, i) * orc_int4_scale(scales, k, group, j, i);
                sum += orc_bf16_to_double(x[(int64_t)b * k + i]) * w;
            }
            if (y_exact)
                y_exact[(int64_t)b * nrows + r] = sum;
            if (y)
                y[(int64_t)b * nrows + r] = orc_bf16_from_double(sum);
        }
    }
}
