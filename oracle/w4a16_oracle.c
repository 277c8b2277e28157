/*
 * CPU oracle for the weight-only int4 (W4A16) linear layer.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path may call, link or
 * execute this file: it is used by tests/, by __graft_entry__.smoke() and by
 * the cpu_baseline / reference leg of bench.py, and nowhere else. It shares no
 * code, header, table or helper with the CUDA library.
 *
 * Plain, slow, single-threaded C99. It computes exactly what the test reference
 * on the vLLM PR #37352 analysis page does ("[vllm] AMD ROCm을 위한 Triton 기반
 * W4A16 커널 도입", section "코드 분석 1. Triton 기반 GEMM 커널 구현 및 검증",
 * the `_w4a16_reference` excerpt), step by step:
 *   1. unpack the int4 nibbles of the [K, N/8] packed weight,
 *   2. take the zero point from the packed [K/G, N/8] zeros, or the constant
 *      zp_bias when no zeros are given,
 *   3. expand scales and zeros along K (group index g = k / G),
 *   4. dequantise in fp32: w = float(q - z) * float(s),
 *   5. matmul in fp32: acc[m][n] = sum over k (ascending) of float(a[m][k]) * w[k][n],
 *   6. cast to the activation dtype (fp16, round to nearest even).
 * The repack follows section "2. 가중치 레이아웃 재포장 (Weight Repacking)" of
 * the same page: checkpoint layout [N, K/8] (8 nibbles per int32 along K) to
 * kernel layout [K, N/8] (8 nibbles per int32 along N).
 *
 * Readings taken where the page is silent:
 *   - nibble j of a 32-bit word (bits 4j..4j+3) holds the element with index
 *     8*c + j along the packed dimension, for weights, zeros and checkpoint;
 *   - nibbles are unsigned 0..15;
 *   - when zeros are given, zp_bias is ignored and the zeros are used as is;
 *   - the fp32 sum runs over k in ascending order, product then add (this
 *     file must be compiled with -ffp-contract=off so no FMA is formed);
 *   - the fp16 cast is IEEE round-to-nearest-even, overflow to +/-inf.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------------- IEEE-754 binary16 <-> binary32 ---------------------------
 * Written from the format definition: 1 sign bit, 5 exponent bits (bias 15),
 * 10 fraction bits; exponent 0 = subnormal (value = frac * 2^-24), exponent 31
 * = inf / NaN.  The binary32 side is built from bits with memcpy. */

static float f32_from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t f32_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

float oracle_half_to_float(uint16_t h)
{
    uint32_t sign = (uint32_t)(h >> 15) & 1u;
    uint32_t e = (uint32_t)(h >> 10) & 0x1fu;
    uint32_t frac = (uint32_t)h & 0x3ffu;
    float mag;
    if (e == 0) {
        /* subnormal or zero: frac * 2^-24, exact in binary32 */
        mag = (float)frac * f32_from_bits(0x33800000u); /* 2^-24 */
    } else if (e == 31) {
        mag = frac ? f32_from_bits(0x7fc00000u) : f32_from_bits(0x7f800000u);
    } else {
        /* (1 + frac/1024) * 2^(e-15): rebuild the binary32 bit pattern */
        mag = f32_from_bits(((e - 15u + 127u) << 23) | (frac << 13));
    }
    return sign ? -mag : mag;
}

uint16_t oracle_float_to_half_rne(float f)
{
    uint32_t u = f32_bits(f);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    uint32_t e32 = (u >> 23) & 0xffu;
    uint32_t m32 = u & 0x7fffffu;
    if (e32 == 0xffu) /* inf or NaN */
        return (uint16_t)(sign | 0x7c00u | (m32 ? 0x200u : 0u));
    if (e32 == 0 && m32 == 0) return sign;
    /* value = sig * 2^(exp2), sig an integer with the implicit bit */
    int64_t sig = (e32 == 0) ? (int64_t)m32 : (int64_t)(m32 | 0x800000u);
    int exp2 = (e32 == 0) ? (1 - 127 - 23) : ((int)e32 - 127 - 23);
    /* Target: a half with 11 significant bits. Find the binary exponent of the
     * value's leading bit, clamp to the subnormal range, and round the integer
     * significand to the half's quantum 2^(qexp) with ties to even. */
    int lead = 63; while (!((sig >> lead) & 1)) --lead;   /* sig has bit `lead` set */
    int vexp = lead + exp2;                                  /* value in [2^vexp, 2^(vexp+1)) */
    int qexp = vexp - 10;                                    /* quantum for a normal half */
    if (qexp < -24) qexp = -24;                              /* subnormal quantum */
    int shift = qexp - exp2;                                 /* bits to drop from sig */
    int64_t q;
    if (shift <= 0) {
        q = sig << (-shift);
    } else if (shift > 62) {
        q = 0;
    } else {
        int64_t keep = sig >> shift;
        int64_t rem = sig - (keep << shift);
        int64_t halfway = (int64_t)1 << (shift - 1);
        if (rem > halfway || (rem == halfway && (keep & 1))) keep += 1;
        q = keep;
    }
    /* q * 2^qexp is the rounded magnitude; q < 2^11 except after a carry */
    if (q == 0) return sign;
    if (q >= 2048) { q >>= 1; qexp += 1; }                   /* carry into next binade */
    if (qexp == -24 && q < 1024) return (uint16_t)(sign | (uint16_t)q);  /* subnormal */
    int ehalf = qexp + 10 + 15;                              /* biased exponent */
    if (ehalf >= 31) return (uint16_t)(sign | 0x7c00u);      /* overflow -> inf */
    return (uint16_t)(sign | (uint16_t)(ehalf << 10) | (uint16_t)(q - 1024));
}

/* ---------------- int4 packing ------------------------------------------- */

static uint8_t nibble(uint32_t word, int j) { return (uint8_t)((word >> (4 * j)) & 0xfu); }

/* Kernel layout [K, N/8]: word (k, c) holds q[k][8c + j] in nibble j. q is [K][N]. */
void oracle_unpack_kn8(const uint32_t* b, int64_t K, int64_t N, uint8_t* q)
{
    for (int64_t k = 0; k < K; ++k)
        for (int64_t n = 0; n < N; ++n)
            q[k * N + n] = nibble(b[k * (N / 8) + n / 8], (int)(n % 8));
}

void oracle_pack_kn8(const uint8_t* q, int64_t K, int64_t N, uint32_t* b)
{
    for (int64_t k = 0; k < K; ++k)
        for (int64_t c = 0; c < N / 8; ++c) {
            uint32_t w = 0;
            for (int j = 0; j < 8; ++j) w |= (uint32_t)(q[k * N + 8 * c + j] & 0xfu) << (4 * j);
            b[k * (N / 8) + c] = w;
        }
}

/* Checkpoint layout [N, K/8]: word (n, c) holds q[8c + j][n] in nibble j. q is [K][N]. */
void oracle_unpack_ct(const uint32_t* ckpt, int64_t N, int64_t K, uint8_t* q)
{
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            q[k * N + n] = nibble(ckpt[n * (K / 8) + k / 8], (int)(k % 8));
}

void oracle_pack_ct(const uint8_t* q, int64_t N, int64_t K, uint32_t* ckpt)
{
    for (int64_t n = 0; n < N; ++n)
        for (int64_t c = 0; c < K / 8; ++c) {
            uint32_t w = 0;
            for (int j = 0; j < 8; ++j) w |= (uint32_t)(q[(8 * c + j) * N + n] & 0xfu) << (4 * j);
            ckpt[n * (K / 8) + c] = w;
        }
}

/* Repack: checkpoint [N, K/8] -> kernel [K, N/8]. Returns 0, or -1 on bad sizes. */
int oracle_repack(const uint32_t* ckpt, int64_t N, int64_t K, uint32_t* out)
{
    if (N <= 0 || K <= 0 || N % 8 || K % 8) return -1;
    uint8_t* q = (uint8_t*)malloc((size_t)(K * N));
    if (!q) return -2;
    oracle_unpack_ct(ckpt, N, K, q);
    oracle_pack_kn8(q, K, N, out);
    free(q);
    return 0;
}

/* Inverse of the repack, used only by the round-trip test. */
int oracle_unrepack(const uint32_t* b, int64_t K, int64_t N, uint32_t* ckpt)
{
    if (N <= 0 || K <= 0 || N % 8 || K % 8) return -1;
    uint8_t* q = (uint8_t*)malloc((size_t)(K * N));
    if (!q) return -2;
    oracle_unpack_kn8(b, K, N, q);
    oracle_pack_ct(q, N, K, ckpt);
    free(q);
    return 0;
}

/* ---------------- checkpoint scales and zeros -> kernel layout ----------------
 * Section "2. 가중치 레이아웃 재포장 (Weight Repacking)" of the PR #37352 page
 * states the layer's layout after loading: weight [K, N/8] and scale [K/G, N].
 * The checkpoint side of the scales and zeros is a reading (the page prints only
 * the weight's): scales are stored per output channel, [N, K/G] fp16 with
 * element (n, g) at n * (K/G) + g; zeros are packed 8 output channels per int32
 * like the kernel's zeros, [N/8, K/G], word (c, g) holding z[8c + j][g] in
 * nibble j. The kernel zeros are [K/G, N/8], word (g, d) holding z[g][8d + j].
 * ngroups = K / G. Both conversions move values only: bit-exact. */
int oracle_ct_scales(const uint16_t* s_ng, int64_t N, int64_t ngroups, uint16_t* s_gn)
{
    if (N <= 0 || ngroups <= 0) return -1;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t g = 0; g < ngroups; ++g)
            s_gn[g * N + n] = s_ng[n * ngroups + g];
    return 0;
}

int oracle_ct_zeros(const uint32_t* z_n8g, int64_t N, int64_t ngroups, uint32_t* z_gn8)
{
    if (N <= 0 || ngroups <= 0 || N % 8) return -1;
    uint8_t* z = (uint8_t*)malloc((size_t)(N * ngroups));   /* z[n][g], one nibble per byte */
    if (!z) return -2;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t g = 0; g < ngroups; ++g)
            z[n * ngroups + g] = nibble(z_n8g[(n / 8) * ngroups + g], (int)(n % 8));
    for (int64_t g = 0; g < ngroups; ++g)
        for (int64_t d = 0; d < N / 8; ++d) {
            uint32_t word = 0;
            for (int j = 0; j < 8; ++j) word |= (uint32_t)z[(8 * d + j) * ngroups + g] << (4 * j);
            z_gn8[g * (N / 8) + d] = word;
        }
    free(z);
    return 0;
}

/* ---------------- GEMM ---------------------------------------------------
 * a      fp16 bits [M, K]
 * b      packed    [K, N/8]
 * s      fp16 bits [K/G, N]
 * z      packed    [K/G, N/8], or NULL for the constant zp_bias
 * cols   the output columns to compute (ncols of them), or NULL for all N
 * acc    (optional) fp32 result before the cast, [M, ncols]
 * out    (optional) fp16 bits [M, ncols]
 * Returns 0, -1 on bad arguments, -2 when out of host memory. */
int oracle_gemm_cols(const uint16_t* a, const uint32_t* b, const uint16_t* s, const uint32_t* z,
                     int64_t M, int64_t N, int64_t K, int32_t G, int32_t zp_bias,
                     const int64_t* cols, int64_t ncols, float* acc, uint16_t* out)
{
    if (M <= 0 || N <= 0 || K <= 0 || G <= 0 || N % 8 || K % G) return -1;
    if (!z && (zp_bias < 0 || zp_bias > 15)) return -1;
    if (!cols) ncols = N;
    for (int64_t i = 0; i < ncols; ++i) {
        int64_t n = cols ? cols[i] : i;
        if (n < 0 || n >= N) return -1;
    }
    /* steps 1-4: dequantised weight w[k][i] for the requested columns, fp32 */
    float* w = (float*)malloc(sizeof(float) * (size_t)(K * ncols));
    float* af = (float*)malloc(sizeof(float) * (size_t)K);
    float* row = (float*)malloc(sizeof(float) * (size_t)ncols);
    if (!w || !af || !row) { free(w); free(af); free(row); return -2; }
    for (int64_t k = 0; k < K; ++k) {
        int64_t g = k / G;                                       /* step 3 */
        for (int64_t i = 0; i < ncols; ++i) {
            int64_t n = cols ? cols[i] : i;
            int q = nibble(b[k * (N / 8) + n / 8], (int)(n % 8)); /* step 1 */
            int zz = z ? nibble(z[g * (N / 8) + n / 8], (int)(n % 8)) : zp_bias; /* step 2 */
            float sc = oracle_half_to_float(s[g * N + n]);
            w[k * ncols + i] = (float)(q - zz) * sc;             /* step 4 */
        }
    }
    /* step 5: fp32 matmul, k ascending for every output element; step 6: cast */
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t k = 0; k < K; ++k) af[k] = oracle_half_to_float(a[m * K + k]);
        for (int64_t i = 0; i < ncols; ++i) row[i] = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            const float ak = af[k];
            const float* wk = w + k * ncols;
            for (int64_t i = 0; i < ncols; ++i) row[i] = row[i] + ak * wk[i];
        }
        for (int64_t i = 0; i < ncols; ++i) {
            if (acc) acc[m * ncols + i] = row[i];
            if (out) out[m * ncols + i] = oracle_float_to_half_rne(row[i]);
        }
    }
    free(w); free(af); free(row);
    return 0;
}

int oracle_gemm(const uint16_t* a, const uint32_t* b, const uint16_t* s, const uint32_t* z,
                int64_t M, int64_t N, int64_t K, int32_t G, int32_t zp_bias,
                float* acc, uint16_t* out)
{
    return oracle_gemm_cols(a, b, s, z, M, N, K, G, zp_bias, (const int64_t*)0, N, acc, out);
}
