/*
 * oracle.c -- plain, slow, single-threaded float64 CPU oracle for token-level
 * sparse Multi-head Latent Attention (MLA) decoding over a paged FP8 KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link or
 * call this file; it exists so that tests, the smoke check and the benchmark's
 * CPU baseline can check the CUDA path against an independent restatement.
 * It shares no code, header, table or constant generator with the CUDA path.
 *
 * Sources (web pages on FlashMLA; cited by page title and section):
 *  [SRC-WALK]  "FlashMLA 注意力内核源码走读：656 字节 KV 缓存背后的完整链路"
 *              sections: 调度 (scheduling), 解码阶段调用示例 (decode call),
 *              数据加载 (data loading / 656-byte layout), 合并与性能账本 (combine).
 *  [SRC-GG]    "deepseek-ai/FlashMLA" (gitgenius repository summary), the
 *              paragraph on the FP8 KV cache format (512 B values, 16 B
 *              scales, 128 B RoPE) and the indices tensor.
 *  [SRC-AL]    "deepseek-ai/FlashMLA" (agentlenshq project page), section
 *              技術的な詳細 (indices: -1 marks an entry the kernel ignores).
 *  [SRC-BLOG]  "FlashMLA：DeepSeek开源的高效MLA解码内核，专为NVIDIA Hopper GPU优化",
 *              sections 主要功能特性 (paged KV cache with block size 64, BF16)
 *              and 基础用法示例 (the dense decode call with causal=True).
 * The method as a whole: MQA with one KV head, d_qk = 576 (512 latent + 64
 * RoPE), d_v = 512 (the latent part), each query token attends to the top-k
 * cache rows its indices list; softmax_scale defaults to 1/sqrt(576); the
 * outputs are o (bf16) and lse (natural log).
 *
 * Parity status: every exported function is pinned by tests under tests/
 * (closed forms, library special cases, brute force, invariants).  None is
 * "parity unpinned".
 *
 * Build: gcc -O2 -std=c99 -fPIC -shared -ffp-contract=off -fno-fast-math
 * (no FMA contraction: every float32 step rounds exactly where written).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define SMO_DQK 576
#define SMO_DV 512
#define SMO_DROPE 64
#define SMO_ROW_BYTES 656
#define SMO_TILE 128          /* quantisation tile: 1 x 128 latent values     */
#define SMO_NTILES 4          /* 512 / 128 scale factors per row              */
#define SMO_BLOCK 64          /* paged-cache block size in tokens             */
#define SMO_SCALE_OFF 512     /* byte offset of the 4 float32 scales          */
#define SMO_ROPE_OFF 528      /* byte offset of the 64 bf16 RoPE values       */
#define SMO_BF16_ROW_BYTES 1152  /* dense BF16 cache row: 576 bf16 values    */

/* ------------------------------------------------------------------------ */
/* Number formats                                                            */
/* ------------------------------------------------------------------------ */

/* float8_e4m3fn decode, written from the format definition: 1 sign bit, 4
 * exponent bits with bias 7, 3 mantissa bits; exponent field 0 encodes the
 * subnormals m * 2^-9; the all-ones pattern S.1111.111 is NaN; there is no
 * infinity, so the largest finite magnitude is 1.75 * 2^8 = 448. */
double smo_e4m3_decode(uint8_t b)
{
    int sign = (b >> 7) & 1;
    int e = (b >> 3) & 0xF;
    int m = b & 0x7;
    double v;
    if (e == 0xF && m == 0x7) return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* Round a non-negative double holding an exact dyadic value to the nearest
 * integer, ties to even (the IEEE default rounding rule). */
static double smo_rne_integer(double v)
{
    double f = floor(v);
    double d = v - f;
    if (d > 0.5) return f + 1.0;
    if (d < 0.5) return f;
    return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

/* float32 -> float8_e4m3fn, round-to-nearest-even with saturation to +-448
 * ("satfinite"); NaN maps to the NaN code.  Written from the format
 * definition: the representable magnitudes are k*2^-9 (k=0..7, subnormal)
 * and q*2^(e-10) for q=8..15, e=1..15 (q=15 at e=15 excluded). */
uint8_t smo_e4m3_encode_satfinite(float xf)
{
    double x = (double)xf;
    uint8_t sign = signbit(xf) ? 0x80 : 0x00;
    double a;
    if (isnan(xf)) return (uint8_t)(sign | 0x7F);
    a = fabs(x);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    if (a < ldexp(1.0, -6)) {
        /* subnormal range: quantum 2^-9; k == 8 carries into the smallest
         * normal, whose encoding is also 8 (exponent field 1, mantissa 0) */
        double k = smo_rne_integer(ldexp(a, 9));
        return (uint8_t)(sign | (uint8_t)k);
    }
    {
        int ex;
        double q;
        int code;
        frexp(a, &ex);            /* a = f * 2^ex, f in [0.5, 1) */
        ex -= 1;                  /* a = g * 2^ex, g in [1, 2)   */
        q = smo_rne_integer(ldexp(a, 3 - ex)); /* in [8, 16] */
        if (q == 16.0) { q = 8.0; ex += 1; }
        code = ((ex + 7) << 3) | ((int)q - 8);
        if (code > 0x7E) code = 0x7E; /* 464 and above rounds past 448 */
        return (uint8_t)(sign | code);
    }
}

/* float32 -> bfloat16 bit pattern, round-to-nearest-even (bfloat16 keeps the
 * top 16 bits of the float32 encoding).  NaN stays NaN (quiet). */
uint16_t smo_bf16_from_float(float x)
{
    uint32_t u;
    uint32_t lsb;
    memcpy(&u, &x, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu) != 0)
        return (uint16_t)((u >> 16) | 0x0040u);
    lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

double smo_bf16_to_double(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static float smo_bf16_to_float(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

static uint16_t smo_load_u16le(const uint8_t* p) { return (uint16_t)(p[0] | (p[1] << 8)); }

static float smo_load_f32le(const uint8_t* p)
{
    uint32_t u = (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24);
    float f;
    memcpy(&f, &u, 4);
    return f;
}

static void smo_store_f32le(uint8_t* p, float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    p[0] = (uint8_t)(u & 0xFF);
    p[1] = (uint8_t)((u >> 8) & 0xFF);
    p[2] = (uint8_t)((u >> 16) & 0xFF);
    p[3] = (uint8_t)((u >> 24) & 0xFF);
}

/* ------------------------------------------------------------------------ */
/* The 656-byte KV row [SRC-WALK 数据加载; SRC-GG FP8 KV cache format]       */
/*   bytes [0,512)   : 512 e4m3 latent values                                */
/*   bytes [512,528) : 4 float32 scales, one per 1x128 tile, little-endian   */
/*   bytes [528,656) : 64 bf16 RoPE values, not quantised, little-endian     */
/* ------------------------------------------------------------------------ */

/* Quantise one token: latent (512 bf16) and rope (64 bf16) -> 656 bytes.
 * Per 128-value tile: amax = max |x| (as float32), scale = amax / 448 in
 * float32, byte = e4m3_rne_satfinite(x / scale) with a float32 division.
 * An all-zero tile gets scale 0 and zero bytes. */
void smo_quantize_token(const uint16_t* latent, const uint16_t* rope, uint8_t* row)
{
    int t, i;
    for (t = 0; t < SMO_NTILES; ++t) {
        float amax = 0.0f;
        float scale;
        for (i = 0; i < SMO_TILE; ++i) {
            float v = fabsf(smo_bf16_to_float(latent[t * SMO_TILE + i]));
            if (v > amax) amax = v;
        }
        scale = amax / 448.0f;
        for (i = 0; i < SMO_TILE; ++i) {
            float x = smo_bf16_to_float(latent[t * SMO_TILE + i]);
            row[t * SMO_TILE + i] = (scale == 0.0f) ? 0 : smo_e4m3_encode_satfinite(x / scale);
        }
        smo_store_f32le(row + SMO_SCALE_OFF + 4 * t, scale);
    }
    for (i = 0; i < SMO_DROPE; ++i) {
        row[SMO_ROPE_OFF + 2 * i] = (uint8_t)(rope[i] & 0xFF);
        row[SMO_ROPE_OFF + 2 * i + 1] = (uint8_t)(rope[i] >> 8);
    }
}

/* Dequantise one row into the 576-wide key: k[i] = bf16(float(e4m3[i]) *
 * scale[i/128]) for i < 512, the product rounded in float32 and then to bf16
 * (round-to-nearest-even); k[512+j] = rope[j].  The value is d_v = k[0..511].
 * Returned as doubles (each is exactly a bf16 value). */
void smo_dequantize_row(const uint8_t* row, double* k)
{
    int i;
    for (i = 0; i < SMO_DV; ++i) {
        float s = smo_load_f32le(row + SMO_SCALE_OFF + 4 * (i / SMO_TILE));
        float p = (float)smo_e4m3_decode(row[i]) * s;  /* float32 product */
        k[i] = smo_bf16_to_double(smo_bf16_from_float(p));
    }
    for (i = 0; i < SMO_DROPE; ++i)
        k[SMO_DV + i] = smo_bf16_to_double(smo_load_u16le(row + SMO_ROPE_OFF + 2 * i));
}

/* ------------------------------------------------------------------------ */
/* Attention over a gathered key set (the plain definition, float64)         */
/* ------------------------------------------------------------------------ */

/* For every head h: s_j = scale * sum_d q[h][d] K[j][d] over the valid rows
 * j; lse = m + ln(sum_j exp(s_j - m)) with m = max_j s_j; the weights are
 * w_j = exp(s_j - lse) and o[h] = sum_j w_j * K[j][0..511].  With no valid
 * row, o = 0 and lse = -inf (and all weights 0).  K rows are 576 wide; V is
 * their first 512 columns (MQA with one shared latent KV head).
 * weights may be NULL; otherwise it receives h_q x n values. */
void smo_attend(int h_q, const double* q, int n, const double* K, const uint8_t* valid,
                double softmax_scale, double* o, double* lse, double* weights)
{
    int h, j, d;
    double* s = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    for (h = 0; h < h_q; ++h) {
        const double* qh = q + (size_t)h * SMO_DQK;
        double* oh = o + (size_t)h * SMO_DV;
        double m = -INFINITY;
        double sum = 0.0;
        double l;
        int any = 0;
        for (d = 0; d < SMO_DV; ++d) oh[d] = 0.0;
        for (j = 0; j < n; ++j) {
            double acc = 0.0;
            if (!valid[j]) continue;
            for (d = 0; d < SMO_DQK; ++d) acc += qh[d] * K[(size_t)j * SMO_DQK + d];
            s[j] = softmax_scale * acc;
            if (s[j] > m) m = s[j];
            any = 1;
        }
        if (!any) {
            lse[h] = -INFINITY;
            if (weights)
                for (j = 0; j < n; ++j) weights[(size_t)h * n + j] = 0.0;
            continue;
        }
        for (j = 0; j < n; ++j)
            if (valid[j]) sum += exp(s[j] - m);
        l = m + log(sum);
        lse[h] = l;
        for (j = 0; j < n; ++j) {
            double w;
            if (!valid[j]) {
                if (weights) weights[(size_t)h * n + j] = 0.0;
                continue;
            }
            w = exp(s[j] - l);
            if (weights) weights[(size_t)h * n + j] = w;
            for (d = 0; d < SMO_DV; ++d) oh[d] += w * K[(size_t)j * SMO_DQK + d];
        }
    }
    free(s);
}

/* ------------------------------------------------------------------------ */
/* One query token of sparse decoding over the paged cache                   */
/* [SRC-WALK 解码阶段调用示例, 数据加载; SRC-AL 技術的な詳細; SRC-BLOG 主要功能特性] */
/* ------------------------------------------------------------------------ */

/* Slot j is valid iff 0 <= idx[j] < seqlen; its cache row is
 * block_table_row[idx/64] * 64 + idx % 64 (block size 64).  Invalid slots are
 * never dereferenced.  q_bf16 holds h_q x 576 bf16 bit patterns.
 * Returns 0, or -1 if a valid slot maps outside the block table or the cache
 * (which a well-formed input never does). */
int smo_sparse_decode_token(int h_q, const uint16_t* q_bf16, const uint8_t* kvcache, int64_t num_blocks,
                            const int32_t* block_table_row, int max_blocks, int32_t seqlen,
                            const int32_t* idx, int topk, double softmax_scale, double* o, double* lse)
{
    int j, i, rc = 0;
    double* q = (double*)malloc(sizeof(double) * (size_t)h_q * SMO_DQK);
    double* K = (double*)malloc(sizeof(double) * (size_t)(topk > 0 ? topk : 1) * SMO_DQK);
    uint8_t* valid = (uint8_t*)malloc((size_t)(topk > 0 ? topk : 1));
    for (i = 0; i < h_q * SMO_DQK; ++i) q[i] = smo_bf16_to_double(q_bf16[i]);
    for (j = 0; j < topk; ++j) {
        int32_t t = idx[j];
        valid[j] = (t >= 0 && t < seqlen) ? 1 : 0;
        if (!valid[j]) continue;
        {
            int32_t blk = t / SMO_BLOCK;
            int64_t phys;
            if (blk >= max_blocks) { rc = -1; valid[j] = 0; continue; }
            phys = (int64_t)block_table_row[blk];
            if (phys < 0 || phys >= num_blocks) { rc = -1; valid[j] = 0; continue; }
            smo_dequantize_row(kvcache + (size_t)(phys * SMO_BLOCK + t % SMO_BLOCK) * SMO_ROW_BYTES,
                               K + (size_t)j * SMO_DQK);
        }
    }
    smo_attend(h_q, q, topk, K, valid, softmax_scale, o, lse, NULL);
    free(q);
    free(K);
    free(valid);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Dense decode: every visible cache token [SRC-BLOG 主要功能特性, 基础用法示例] */
/* ------------------------------------------------------------------------ */

/* A BF16 cache row holds the 576-wide key as 576 little-endian bf16 values
 * (latent then RoPE); nothing is quantised. */
void smo_bf16_row(const uint8_t* row, double* k)
{
    int i;
    for (i = 0; i < SMO_DQK; ++i) k[i] = smo_bf16_to_double(smo_load_u16le(row + 2 * i));
}

/* Cache tokens visible to query token t of s_q new tokens of a request whose
 * cache holds seqlen tokens.  The s_q tokens are the last s_q positions of the
 * cache; with the causal mask token t sees positions 0 .. seqlen - s_q + t,
 * without it every position.  Clamped to [0, seqlen]. */
int32_t smo_dense_visible_len(int32_t seqlen, int s_q, int t, int causal)
{
    int64_t len = causal ? (int64_t)seqlen - (s_q - 1 - t) : (int64_t)seqlen;
    if (len < 0) len = 0;
    if (len > seqlen) len = seqlen;
    return (int32_t)len;
}

/* One query token of dense decoding: attention over cache positions
 * 0 .. len-1 of the request, row of position i = block_table_row[i/64] * 64 +
 * i % 64.  kv_format 0: 656-byte FP8 rows (dequantised as for the sparse
 * decode); 1: 1152-byte BF16 rows.  Returns 0, or -1 if a position maps
 * outside the block table or the cache (its token is then left out). */
int smo_dense_decode_token(int h_q, const uint16_t* q_bf16, const uint8_t* kvcache, int kv_format,
                           int64_t num_blocks, const int32_t* block_table_row, int max_blocks, int32_t len,
                           double softmax_scale, double* o, double* lse)
{
    int i, rc = 0;
    const size_t row_bytes = kv_format ? SMO_BF16_ROW_BYTES : SMO_ROW_BYTES;
    const int n = len > 0 ? len : 0;
    double* q = (double*)malloc(sizeof(double) * (size_t)h_q * SMO_DQK);
    double* K = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * SMO_DQK);
    uint8_t* valid = (uint8_t*)malloc((size_t)(n > 0 ? n : 1));
    for (i = 0; i < h_q * SMO_DQK; ++i) q[i] = smo_bf16_to_double(q_bf16[i]);
    for (i = 0; i < n; ++i) {
        int32_t blk = i / SMO_BLOCK;
        int64_t phys;
        valid[i] = 0;
        if (blk >= max_blocks) { rc = -1; continue; }
        phys = (int64_t)block_table_row[blk];
        if (phys < 0 || phys >= num_blocks) { rc = -1; continue; }
        {
            const uint8_t* row = kvcache + (size_t)(phys * SMO_BLOCK + i % SMO_BLOCK) * row_bytes;
            if (kv_format) smo_bf16_row(row, K + (size_t)i * SMO_DQK);
            else smo_dequantize_row(row, K + (size_t)i * SMO_DQK);
        }
        valid[i] = 1;
    }
    smo_attend(h_q, q, n, K, valid, softmax_scale, o, lse, NULL);
    free(q);
    free(K);
    free(valid);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* LSE-weighted combine of split partials [SRC-WALK 合并与性能账本]          */
/* ------------------------------------------------------------------------ */

/* Given nsplit partial results (o_s, lse_s) of the same heads over disjoint
 * parts of the slots: lse = ln(sum_s exp(lse_s)), o = sum_s exp(lse_s - lse) o_s.
 * If every lse_s is -inf the result is o = 0, lse = -inf. */
void smo_combine(int nsplit, int h_q, const double* o_parts, const double* lse_parts, double* o, double* lse)
{
    int h, s, d;
    for (h = 0; h < h_q; ++h) {
        double m = -INFINITY, sum = 0.0, l;
        double* oh = o + (size_t)h * SMO_DV;
        for (d = 0; d < SMO_DV; ++d) oh[d] = 0.0;
        for (s = 0; s < nsplit; ++s) {
            double v = lse_parts[(size_t)s * h_q + h];
            if (v > m) m = v;
        }
        if (m == -INFINITY) { lse[h] = -INFINITY; continue; }
        for (s = 0; s < nsplit; ++s) sum += exp(lse_parts[(size_t)s * h_q + h] - m);
        l = m + log(sum);
        lse[h] = l;
        for (s = 0; s < nsplit; ++s) {
            double w = exp(lse_parts[(size_t)s * h_q + h] - l);
            const double* os = o_parts + ((size_t)s * h_q + h) * SMO_DV;
            for (d = 0; d < SMO_DV; ++d) oh[d] += w * os[d];
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Tile-scheduler metadata [SRC-WALK 调度]                                   */
/* ------------------------------------------------------------------------ */

/* The pages say only that a small kernel spreads (request, KV-range) work
 * units evenly over all SMs before the main kernel, and that the main kernel
 * follows that table without arbitration.  Reading used here (sparse mode):
 * every request r in [0, R) has n index tiles (n = ceil(topk / 64)); the R*n
 * tiles are laid out in (request, tile) order and cut into P consecutive
 * ranges of L = ceil(R*n / P) tiles.  Part p covers [p*L, min((p+1)*L, R*n)).
 *
 * first(r) = floor(r*n / L), last(r) = floor(((r+1)*n - 1) / L);
 * S_r = last(r) - first(r) + 1 is the number of splits of request r;
 * num_splits[0] = 0, num_splits[r+1] = num_splits[r] + S_r.
 * sched_meta[p] = { begin_r, begin_tile, end_r, end_tile, first_slot,
 *                   is_empty, 0, 0 }
 * where (begin_r, begin_tile) = divmod(p*L, n), (end_r, end_tile) =
 * divmod(min((p+1)*L, R*n), n) is the exclusive end, and first_slot =
 * num_splits[begin_r] + p - first(begin_r) is the split slot of the part's
 * first request.  Empty parts (p*L >= R*n) are {0,0,0,0,0,1,0,0}.
 * Returns 0, or -1 on invalid arguments. */
int smo_sched_meta(int R, int n, int P, int32_t* sched_meta, int32_t* num_splits)
{
    int64_t total, L;
    int r, p;
    if (R < 0 || n < 1 || P < 1) return -1;
    total = (int64_t)R * n;
    L = total > 0 ? (total + P - 1) / P : 1;
    num_splits[0] = 0;
    for (r = 0; r < R; ++r) {
        int64_t first = ((int64_t)r * n) / L;
        int64_t last = ((int64_t)(r + 1) * n - 1) / L;
        num_splits[r + 1] = num_splits[r] + (int32_t)(last - first + 1);
    }
    for (p = 0; p < P; ++p) {
        int32_t* m = sched_meta + (size_t)p * 8;
        int64_t g0 = (int64_t)p * L;
        int64_t g1 = (int64_t)(p + 1) * L;
        int i;
        for (i = 0; i < 8; ++i) m[i] = 0;
        if (g0 >= total) { m[5] = 1; continue; }
        if (g1 > total) g1 = total;
        m[0] = (int32_t)(g0 / n);
        m[1] = (int32_t)(g0 % n);
        m[2] = (int32_t)(g1 / n);
        m[3] = (int32_t)(g1 % n);
        m[4] = num_splits[m[0]] + p - (int32_t)((((int64_t)m[0]) * n) / L);
        m[5] = 0;
    }
    return 0;
}

/* The same division of work when requests have different numbers of tiles
 * (dense decode: n[r] = ceil(visible tokens / 64), at least 1, so every
 * request has a tile and gets its (o, lse) written).  tile_prefix[r] is the
 * number of tiles before request r (length R + 1); the G = tile_prefix[R]
 * tiles in (request, tile) order are cut into P ranges of L = ceil(G / P);
 * part p covers global tiles [p L, min((p+1) L, G)).  A request's parts are
 * first(r) = tile_prefix[r] / L .. last(r) = (tile_prefix[r+1] - 1) / L, and
 * sched_meta / num_splits have the meaning of smo_sched_meta with tile
 * positions counted within each request.  Returns -1 for a tile count < 1. */
int smo_sched_meta_varlen(int R, const int32_t* n, int P, int32_t* sched_meta, int32_t* num_splits,
                          int32_t* tile_prefix)
{
    int64_t total, L;
    int r, p;
    if (R < 0 || P < 1) return -1;
    tile_prefix[0] = 0;
    for (r = 0; r < R; ++r) {
        if (n[r] < 1) return -1;
        tile_prefix[r + 1] = tile_prefix[r] + n[r];
    }
    total = tile_prefix[R];
    L = total > 0 ? (total + P - 1) / P : 1;
    num_splits[0] = 0;
    for (r = 0; r < R; ++r) {
        int64_t first = (int64_t)tile_prefix[r] / L;
        int64_t last = ((int64_t)tile_prefix[r + 1] - 1) / L;
        num_splits[r + 1] = num_splits[r] + (int32_t)(last - first + 1);
    }
    for (p = 0; p < P; ++p) {
        int32_t* m = sched_meta + (size_t)p * 8;
        int64_t g0 = (int64_t)p * L;
        int64_t g1 = (int64_t)(p + 1) * L;
        int i, rb, re;
        for (i = 0; i < 8; ++i) m[i] = 0;
        if (g0 >= total) { m[5] = 1; continue; }
        if (g1 > total) g1 = total;
        /* the request holding global tile g0: the last r with tile_prefix[r] <= g0 */
        rb = 0;
        while (rb + 1 < R && tile_prefix[rb + 1] <= g0) ++rb;
        /* the exclusive end: request R with tile 0 when g1 reaches the total */
        if (g1 == total) {
            re = R;
        } else {
            re = rb;
            while (re + 1 < R && tile_prefix[re + 1] <= g1) ++re;
        }
        m[0] = rb;
        m[1] = (int32_t)(g0 - tile_prefix[rb]);
        m[2] = re;
        m[3] = (re == R) ? 0 : (int32_t)(g1 - tile_prefix[re]);
        m[4] = num_splits[rb] + p - (int32_t)((int64_t)tile_prefix[rb] / L);
        m[5] = 0;
    }
    return 0;
}
