// Scalar CPU oracle for block-quantized W4A8 matmul (Q4_0 weights x Q8_0 activations)
// and its affine 4-, 6- and 8-bit variants.
//
// TEST INFRASTRUCTURE ONLY. Nothing on the product path may link, load or call this
// file; only the tests, the smoke check and the benchmark's CPU-baseline leg use it.
// It shares no code, header, table or constant with the CUDA library.
//
// Every routine is written for a reader checking it by eye against the definitions:
// plain loops, one element at a time, in the order the definitions state. Built with
// -O2 -ffp-contract=off so that no multiply-add is fused (each f32 operation rounds
// on its own, as the definitions require).
//
// Sources (pages on the subject):
//  * tract PR #2432 "W4A8 (Q4_0 int8-dot) path for block_quant", section "The kernel":
//    Q4_0 4-bit weights stored N x K with one scale per 32-block, activations
//    re-quantised to int8 per block, integer block dot, per-block f32 rescale.
//  * The Q4_0 / Q8_0 bit-level encodings (fp16 weight scale d, codes q in [0,15],
//    w = d*(q-8), low nibbles = elements 0-15 and high nibbles = 16-31 of a block;
//    activation d = amax/127 in f32, q = round-half-away(x*(1/d)) clamped to +-127).
//  * C-Kernel-Engine gemm_kernels_q4k.c, "GEMV: y = W @ x" and "Backward Pass: Gradient
//    w.r.t. Input": Q4_K weights (super-blocks of 256 with fp16 d and dmin and eight
//    6-bit sub-block scales and mins, w = d*sc*q - dmin*m per 32-element sub-block) times
//    FP32 activations, and the input gradient dX = W^T dY with the weights frozen.
//  * MLX PR #4802 "mx.qqmm ... mode=affine": affine 4-, 6- and 8-bit weights with a
//    per-group scale and bias; the int8 MMA runs on the original codes and the scale and
//    bias are applied afterwards (scale = (max-min)/(2^bits - 1), bias = min per group).
//
// Readings where the sources leave a step open are marked "Reading:".

#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

// Runs f(e) for every e in [0, count), the range split into contiguous chunks over
// `nthreads` host threads. Each output element is computed by exactly one call, so the
// result does not depend on the thread count.
template <class F>
static void parallel_over(int64_t count, int nthreads, F f) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads == 1 || count < 2) {
        for (int64_t e = 0; e < count; ++e) f(e);
        return;
    }
    std::vector<std::thread> pool;
    for (int t = 0; t < nthreads; ++t) {
        const int64_t e0 = count * t / nthreads, e1 = count * (t + 1) / nthreads;
        if (e1 > e0) pool.emplace_back([=]() { for (int64_t e = e0; e < e1; ++e) f(e); });
    }
    for (auto& th : pool) th.join();
}

extern "C" {

// ---------------------------------------------------------------------------------
// O1. IEEE-754 conversions, written from the bit layout (round to nearest, ties to
//     even). fp16: 1 sign, 5 exponent, 10 fraction bits. bf16: 1 sign, 8 exponent,
//     7 fraction bits. Both have subnormals; overflow goes to infinity.
// ---------------------------------------------------------------------------------

// Round the non-negative integer `sig` right by `shift` bits, ties to even.
static uint64_t round_shift_rne(uint64_t sig, int shift) {
    if (shift <= 0) return sig << (-shift);
    if (shift >= 64) return 0;
    uint64_t q = sig >> shift;
    uint64_t rem = sig & ((uint64_t(1) << shift) - 1);
    uint64_t half = uint64_t(1) << (shift - 1);
    if (rem > half || (rem == half && (q & 1))) q += 1;
    return q;
}

// Shared narrowing routine: `frac_bits` fraction bits, exponent bias `bias`, exponent
// field width `exp_bits`. Returns the narrow bit pattern.
static uint32_t narrow_rne(float f, int frac_bits, int exp_bits, int bias) {
    uint32_t x;
    std::memcpy(&x, &f, 4);
    const uint32_t sign = x >> 31;
    const uint32_t e = (x >> 23) & 0xFF;
    const uint32_t m = x & 0x7FFFFF;
    const uint32_t exp_max = (1u << exp_bits) - 1;
    const uint32_t sign_out = sign << (frac_bits + exp_bits);
    if (e == 0xFF) {  // infinity or NaN
        if (m == 0) return sign_out | (exp_max << frac_bits);
        return sign_out | (exp_max << frac_bits) | (1u << (frac_bits - 1));  // quiet NaN
    }
    // value = sig * 2^E exactly
    uint64_t sig;
    int E;
    if (e == 0) { sig = m; E = -149; } else { sig = m | 0x800000u; E = int(e) - 150; }
    if (sig == 0) return sign_out;
    int top = 63 - __builtin_clzll(sig);       // floor(log2(sig))
    int lg = E + top;                           // floor(log2(value))
    int min_normal_lg = 1 - bias;               // exponent of the smallest normal
    int q_exp = lg - frac_bits;                 // quantum of the value's binade
    int q_min = min_normal_lg - frac_bits;      // quantum of the subnormal range
    if (q_exp < q_min) q_exp = q_min;
    uint64_t r = round_shift_rne(sig, q_exp - E);   // value ~= r * 2^q_exp
    if (r == 0) return sign_out;
    if (r >= (uint64_t(2) << frac_bits)) { r >>= 1; q_exp += 1; }  // rounded up a binade
    uint32_t out;
    if (r < (uint64_t(1) << frac_bits)) {
        out = uint32_t(r);                      // subnormal (q_exp == q_min)
    } else {
        int biased = q_exp + frac_bits + bias;  // r in [2^f, 2^(f+1))
        if (biased >= int(exp_max)) return sign_out | (exp_max << frac_bits);  // inf
        out = (uint32_t(biased) << frac_bits) | uint32_t(r - (uint64_t(1) << frac_bits));
    }
    return sign_out | out;
}

uint16_t orc_f32_to_f16(float f) { return uint16_t(narrow_rne(f, 10, 5, 15)); }
uint16_t orc_f32_to_bf16(float f) { return uint16_t(narrow_rne(f, 7, 8, 127)); }

static float widen(uint32_t h, int frac_bits, int exp_bits, int bias) {
    const uint32_t sign = (h >> (frac_bits + exp_bits)) & 1;
    const uint32_t e = (h >> frac_bits) & ((1u << exp_bits) - 1);
    const uint32_t m = h & ((1u << frac_bits) - 1);
    const uint32_t exp_max = (1u << exp_bits) - 1;
    double v;
    if (e == exp_max) v = m ? NAN : INFINITY;
    else if (e == 0) v = std::ldexp(double(m), 1 - bias - frac_bits);
    else v = std::ldexp(double(m | (1u << frac_bits)), int(e) - bias - frac_bits);
    float r = float(v);  // exact: every fp16/bf16 value is an f32 value
    return sign ? -r : r;
}

float orc_f16_to_f32(uint16_t h) { return widen(h, 10, 5, 15); }
float orc_bf16_to_f32(uint16_t h) { return widen(h, 7, 8, 127); }

void orc_f32_to_f16_array(const float* in, uint16_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_f32_to_f16(in[i]);
}
void orc_f32_to_bf16_array(const float* in, uint16_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_f32_to_bf16(in[i]);
}
void orc_f16_to_f32_array(const uint16_t* in, float* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_f16_to_f32(in[i]);
}
void orc_bf16_to_f32_array(const uint16_t* in, float* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_bf16_to_f32(in[i]);
}

// ---------------------------------------------------------------------------------
// O2. Q4_0 weight pack. W is N x K row-major f32 (the "4-bit, N x K" weight of the
//     tract page). For row n and block b (elements x_0..x_31 = W[n][32b .. 32b+31]):
//       mx  = the element of largest magnitude (first one wins on ties)
//       d   = mx / -8                     (f32)
//       id  = d != 0 ? 1/d : 0            (f32)
//       q_i = min(15, trunc(x_i*id + 8.5)), multiply and add rounded separately
//       scale stored as fp16(d); byte j of the block = q_j | q_{j+16} << 4.
//     Dequantised weight: fp16(d) * (q - 8).
//     Reading: the pages fix only w = d*(q-8) with q in [0,15]; dividing the signed
//     largest-magnitude element by -8 is the only choice under which that element
//     reaches code 0 (the end of the grid), so the whole 16-level grid is used.
//     Reading: the codes use the f32 d (before its fp16 rounding).
// ---------------------------------------------------------------------------------
void orc_pack_q4_0(const float* w, int N, int K, uint8_t* qs, uint16_t* d_out) {
    const int B = K / 32;
    for (int n = 0; n < N; ++n) {
        for (int b = 0; b < B; ++b) {
            const float* x = w + int64_t(n) * K + 32 * b;
            float amax = 0.0f, mx = 0.0f;
            for (int i = 0; i < 32; ++i) {
                float a = std::fabs(x[i]);
                if (a > amax) { amax = a; mx = x[i]; }
            }
            float d = mx / -8.0f;
            float id = (d != 0.0f) ? 1.0f / d : 0.0f;
            int q[32];
            for (int i = 0; i < 32; ++i) {
                float t = x[i] * id;
                t = t + 8.5f;
                int qi = int(t);  // truncation; t >= 0.5 - ulp here, so this is floor
                if (qi > 15) qi = 15;
                if (qi < 0) qi = 0;
                q[i] = qi;
            }
            uint8_t* out = qs + int64_t(n) * (K / 2) + 16 * b;
            for (int j = 0; j < 16; ++j) out[j] = uint8_t(q[j] | (q[j + 16] << 4));
            d_out[int64_t(n) * B + b] = orc_f32_to_f16(d);
        }
    }
}

// Code of element k of row n of a packed Q4_0 matrix (0..15).
static int q4_0_code(const uint8_t* qs, int K, int n, int k) {
    const int b = k / 32, j = k % 32;
    uint8_t byte = qs[int64_t(n) * (K / 2) + 16 * b + (j & 15)];
    return (j < 16) ? (byte & 0x0F) : (byte >> 4);
}

// Dequantise the whole packed matrix to f64 (for brute-force checks).
void orc_dequant_q4_0(const uint8_t* qs, const uint16_t* d, int N, int K, double* w_out) {
    const int B = K / 32;
    for (int n = 0; n < N; ++n)
        for (int k = 0; k < K; ++k)
            w_out[int64_t(n) * K + k] =
                double(orc_f16_to_f32(d[int64_t(n) * B + k / 32])) * double(q4_0_code(qs, K, n, k) - 8);
}

// ---------------------------------------------------------------------------------
// O3. Q8_0 activation quantisation. x is M x K row-major (f32, or bf16 widened
//     exactly). For row m and block b:
//       amax = max |x_i|;  d = amax / 127 (f32, stored as f32);  id = d != 0 ? 1/d : 0
//       q_i  = clamp(round_half_away(x_i * id), -127, 127);  s = sum of q_i (int32)
//     Reading: the scale is kept in f32 as stated, not narrowed to fp16.
// ---------------------------------------------------------------------------------
void orc_quant_act_q8_0(const float* x, int M, int K, int8_t* qx, float* dx, int32_t* sx) {
    const int B = K / 32;
    for (int m = 0; m < M; ++m) {
        for (int b = 0; b < B; ++b) {
            const float* v = x + int64_t(m) * K + 32 * b;
            float amax = 0.0f;
            for (int i = 0; i < 32; ++i) {
                float a = std::fabs(v[i]);
                if (a > amax) amax = a;
            }
            float d = amax / 127.0f;
            float id = (d != 0.0f) ? 1.0f / d : 0.0f;
            int32_t s = 0;
            for (int i = 0; i < 32; ++i) {
                float t = v[i] * id;
                float r = std::round(t);  // halfway cases away from zero
                int qi = int(r);
                if (qi > 127) qi = 127;
                if (qi < -127) qi = -127;
                qx[int64_t(m) * K + 32 * b + i] = int8_t(qi);
                s += qi;
            }
            dx[int64_t(m) * B + b] = d;
            if (sx) sx[int64_t(m) * B + b] = s;
        }
    }
}

void orc_dequant_q8_0(const int8_t* qx, const float* dx, int M, int K, double* x_out) {
    const int B = K / 32;
    for (int m = 0; m < M; ++m)
        for (int k = 0; k < K; ++k)
            x_out[int64_t(m) * K + k] = double(dx[int64_t(m) * B + k / 32]) * double(qx[int64_t(m) * K + k]);
}

// ---------------------------------------------------------------------------------
// O4. Q4_0 x Q8_0 contraction, y = x . W^T (y is M x N).
//       D[m,n,b] = sum_j (q_w - 8) * q_x      (exact int32, |D| <= 32512)
//       term     = f32(d_w) * d_x * D        (evaluated in f64: 11+24+16 bits <= 53,
//                                              so every term is exact)
//       y        = sum_b term (f64),  T = sum_b |term|  (the tolerance scale)
// ---------------------------------------------------------------------------------
static void gemm_q4_0_one(int K, int m, int n, const int8_t* qx, const float* dx,
                          const uint8_t* qs, const uint16_t* d, double* y, double* T) {
    const int B = K / 32;
    double acc = 0.0, tabs = 0.0;
    for (int b = 0; b < B; ++b) {
        int32_t D = 0;
        for (int j = 0; j < 32; ++j) {
            const int k = 32 * b + j;
            D += (q4_0_code(qs, K, n, k) - 8) * int32_t(qx[int64_t(m) * K + k]);
        }
        double term = double(orc_f16_to_f32(d[int64_t(n) * B + b])) * double(dx[int64_t(m) * B + b]) * double(D);
        acc += term;
        tabs += std::fabs(term);
    }
    *y = acc;
    if (T) *T = tabs;
}

// Full output; output elements are split over `nthreads` host threads.
void orc_gemm_q4_0(int M, int N, int K, const int8_t* qx, const float* dx, const uint8_t* qs,
                   const uint16_t* d, double* y, double* T, int nthreads) {
    auto one = [&](int64_t e) {
        const int m = int(e / N), n = int(e % N);
        gemm_q4_0_one(K, m, n, qx, dx, qs, d, y + e, T ? T + e : nullptr);
    };
    parallel_over(int64_t(M) * N, nthreads, one);
}

// Selected output elements only: (ms[i], ns[i]) for i < count.
void orc_gemm_q4_0_sampled(int K, int count, const int32_t* ms, const int32_t* ns, const int8_t* qx,
                           const float* dx, const uint8_t* qs, const uint16_t* d, double* y, double* T) {
    for (int i = 0; i < count; ++i)
        gemm_q4_0_one(K, ms[i], ns[i], qx, dx, qs, d, y + i, T ? T + i : nullptr);
}

// The same contraction with the per-block rescale done in f32, summed in block order
// (fl(fl(d_w*d_x) * float(D)) added to an f32 running sum): the "per-block f32
// rescale" of the tract page. Used to show that plain f32 accumulation meets the
// tolerance the GPU path is held to.
void orc_gemm_q4_0_f32(int M, int N, int K, const int8_t* qx, const float* dx, const uint8_t* qs,
                       const uint16_t* d, float* y) {
    const int B = K / 32;
    for (int m = 0; m < M; ++m)
        for (int n = 0; n < N; ++n) {
            float acc = 0.0f;
            for (int b = 0; b < B; ++b) {
                int32_t D = 0;
                for (int j = 0; j < 32; ++j) {
                    const int k = 32 * b + j;
                    D += (q4_0_code(qs, K, n, k) - 8) * int32_t(qx[int64_t(m) * K + k]);
                }
                float s = orc_f16_to_f32(d[int64_t(n) * B + b]) * dx[int64_t(m) * B + b];
                float t = s * float(D);
                acc = acc + t;
            }
            y[int64_t(m) * N + n] = acc;
        }
}

// ---------------------------------------------------------------------------------
// O5. Affine weight pack with `bits`-bit codes (4, 6 or 8), per row n and group g of
//     `group` (32, 64 or 128) consecutive elements along K:
//       mn = min, mx = max (f32)
//       s  = bf16((mx - mn) / (2^bits - 1)),  b = bf16(mn)
//       q  = s != 0 ? clamp(round_half_away((w - b) / s), 0, 2^bits - 1) : 0   (f32 ops,
//            using the stored bf16 s and b)
//     Codes of a row form a little-endian bit stream: element k at bits [bits*k,
//     bits*k + bits) of the row's K*bits/8 bytes (for 4 bits: eight codes per 32-bit
//     little-endian word, element k at bits 4*(k%8) of word k/8). Dequantised weight:
//     s*q + b.
//     Reading: the codes are computed against the stored (bf16) scale and bias so that
//     s*q + b is the nearest grid point the kernel can reconstruct; the clamp is needed
//     because rounding s and b to bf16 can push an end code to -1 or 2^bits.
//     Reading: the pages name 6- and 8-bit codes but not their packing; the bit stream
//     is the one layout that contains the 4-bit word layout as its special case.
// ---------------------------------------------------------------------------------
static int64_t affine_row_bytes(int K, int bits) { return int64_t(K) * bits / 8; }

static void put_code(uint8_t* row, int bits, int k, int q) {
    for (int i = 0; i < bits; ++i) {
        const int64_t bit = int64_t(k) * bits + i;
        if ((q >> i) & 1) row[bit / 8] |= uint8_t(1u << (bit % 8));
    }
}

static int affine_code(const uint8_t* q, int K, int bits, int n, int k) {
    const uint8_t* row = q + int64_t(n) * affine_row_bytes(K, bits);
    int v = 0;
    for (int i = 0; i < bits; ++i) {
        const int64_t bit = int64_t(k) * bits + i;
        v |= ((row[bit / 8] >> (bit % 8)) & 1) << i;
    }
    return v;
}

void orc_pack_affine_bits(const float* w, int N, int K, int group, int bits, uint8_t* q_out, uint16_t* scale,
                          uint16_t* bias) {
    const int G = K / group;
    const int qmax = (1 << bits) - 1;
    for (int n = 0; n < N; ++n) {
        uint8_t* row = q_out + int64_t(n) * affine_row_bytes(K, bits);
        for (int64_t i = 0; i < affine_row_bytes(K, bits); ++i) row[i] = 0;
        for (int g = 0; g < G; ++g) {
            const float* x = w + int64_t(n) * K + int64_t(g) * group;
            float mn = x[0], mx = x[0];
            for (int i = 1; i < group; ++i) {
                if (x[i] < mn) mn = x[i];
                if (x[i] > mx) mx = x[i];
            }
            float range = mx - mn;
            float sf32 = range / float(qmax);
            uint16_t s_bits = orc_f32_to_bf16(sf32);
            uint16_t b_bits = orc_f32_to_bf16(mn);
            float s = orc_bf16_to_f32(s_bits), b = orc_bf16_to_f32(b_bits);
            for (int i = 0; i < group; ++i) {
                int qi = 0;
                if (s != 0.0f) {
                    float t = x[i] - b;
                    t = t / s;
                    qi = int(std::round(t));
                    if (qi > qmax) qi = qmax;
                    if (qi < 0) qi = 0;
                }
                put_code(row, bits, g * group + i, qi);
            }
            scale[int64_t(n) * G + g] = s_bits;
            bias[int64_t(n) * G + g] = b_bits;
        }
    }
}

void orc_dequant_affine_bits(const uint8_t* q, const uint16_t* scale, const uint16_t* bias, int N, int K,
                             int group, int bits, double* w_out) {
    const int G = K / group;
    for (int n = 0; n < N; ++n)
        for (int k = 0; k < K; ++k) {
            double s = orc_bf16_to_f32(scale[int64_t(n) * G + k / group]);
            double b = orc_bf16_to_f32(bias[int64_t(n) * G + k / group]);
            w_out[int64_t(n) * K + k] = s * double(affine_code(q, K, bits, n, k)) + b;
        }
}

// ---------------------------------------------------------------------------------
// O6. Affine contraction on the original codes. For activation block b (32 wide),
//     inside weight group g = 32b / group:
//       D = sum_j q * q_x  (int32, |D| <= 255*127*32),  S = sum_j q_x  (the Q8_0 block sum)
//       term = d_x*s_g*D + d_x*b_g*S   (each product exact in f64: 8 + 24 + 20 bits)
//       y = sum of terms (f64), T = sum(|d_x s D| + |d_x b S|)
//     This is the expansion of sum_k (s q_k + b) (d_x q_x,k) over the block.
// ---------------------------------------------------------------------------------
static void gemm_affine_one(int K, int group, int bits, int m, int n, const int8_t* qx, const float* dx,
                            const int32_t* sx, const uint8_t* q, const uint16_t* scale,
                            const uint16_t* bias, double* y, double* T) {
    const int B = K / 32, G = K / group;
    double acc = 0.0, tabs = 0.0;
    for (int b = 0; b < B; ++b) {
        const int g = (32 * b) / group;
        int32_t D = 0;
        for (int j = 0; j < 32; ++j) {
            const int k = 32 * b + j;
            D += affine_code(q, K, bits, n, k) * int32_t(qx[int64_t(m) * K + k]);
        }
        const int32_t S = sx[int64_t(m) * B + b];
        const double dxv = dx[int64_t(m) * B + b];
        const double s = orc_bf16_to_f32(scale[int64_t(n) * G + g]);
        const double bb = orc_bf16_to_f32(bias[int64_t(n) * G + g]);
        double t1 = dxv * s * double(D);
        double t2 = dxv * bb * double(S);
        acc += t1 + t2;
        tabs += std::fabs(t1) + std::fabs(t2);
    }
    *y = acc;
    if (T) *T = tabs;
}

void orc_gemm_affine_bits(int M, int N, int K, int group, int bits, const int8_t* qx, const float* dx,
                          const int32_t* sx, const uint8_t* q, const uint16_t* scale, const uint16_t* bias,
                          double* y, double* T, int nthreads) {
    auto one = [&](int64_t e) {
        const int m = int(e / N), n = int(e % N);
        gemm_affine_one(K, group, bits, m, n, qx, dx, sx, q, scale, bias, y + e, T ? T + e : nullptr);
    };
    parallel_over(int64_t(M) * N, nthreads, one);
}

void orc_gemm_affine_bits_sampled(int K, int group, int bits, int count, const int32_t* ms, const int32_t* ns,
                                  const int8_t* qx, const float* dx, const int32_t* sx, const uint8_t* q,
                                  const uint16_t* scale, const uint16_t* bias, double* y, double* T) {
    for (int i = 0; i < count; ++i)
        gemm_affine_one(K, group, bits, ms[i], ns[i], qx, dx, sx, q, scale, bias, y + i, T ? T + i : nullptr);
}

// ---------------------------------------------------------------------------------
// O7. Q4_K weights (C-Kernel-Engine gemm_kernels_q4k.c, "GEMV: y = W @ x"; the page
//     follows the llama.cpp Q4_K layout). W is N rows x K/256 super-blocks of 144 bytes:
//       bytes 0-1  d (fp16), bytes 2-3 dmin (fp16), bytes 4-15 the packed 6-bit scales
//       sc[0..7] and mins m[0..7], bytes 16-143 qs[0..127] (codes 0..15).
//     Within a super-block, the 64 elements 64i..64i+63 (i = 0..3) use qs[32i..32i+31]:
//     element 64i + l (l < 32) is the low nibble of qs[32i + l] with sub-block 2i, element
//     64i + 32 + l the high nibble with sub-block 2i + 1. Weight: w = d*sc[j]*q - dmin*m[j]
//     for sub-block j.
//     Reading (the page calls unpack_q4_k_scales without printing it; it names the llama.cpp
//     layout): for j < 4, sc[j] = s[j] & 63 and m[j] = s[j+4] & 63; for j >= 4,
//     sc[j] = (s[j+4] & 15) | ((s[j-4] >> 6) << 4) and m[j] = (s[j+4] >> 4) | ((s[j] >> 6) << 4),
//     s being the 12 scale bytes.
// ---------------------------------------------------------------------------------
void orc_q4_k_unpack_scales(const uint8_t* s, uint8_t* sc, uint8_t* m) {
    for (int j = 0; j < 8; ++j) {
        if (j < 4) {
            sc[j] = uint8_t(s[j] & 63);
            m[j] = uint8_t(s[j + 4] & 63);
        } else {
            sc[j] = uint8_t((s[j + 4] & 15) | ((s[j - 4] >> 6) << 4));
            m[j] = uint8_t((s[j + 4] >> 4) | ((s[j] >> 6) << 4));
        }
    }
}

// Weight of element k of row n, exact in f64 (d*sc*q: 11 + 6 + 4 bits; dmin*m: 11 + 6).
static double q4_k_weight(const uint8_t* W, int K, int n, int k) {
    const int64_t row_bytes = int64_t(K / 256) * 144;
    const uint8_t* blk = W + int64_t(n) * row_bytes + int64_t(k / 256) * 144;
    uint16_t d_bits, dmin_bits;
    std::memcpy(&d_bits, blk, 2);
    std::memcpy(&dmin_bits, blk + 2, 2);
    uint8_t sc[8], m[8];
    orc_q4_k_unpack_scales(blk + 4, sc, m);
    const int e = k % 256;
    const int i = e / 64, r = e % 64;
    int q, j;
    if (r < 32) {
        q = blk[16 + 32 * i + r] & 15;
        j = 2 * i;
    } else {
        q = blk[16 + 32 * i + (r - 32)] >> 4;
        j = 2 * i + 1;
    }
    return double(orc_f16_to_f32(d_bits)) * double(sc[j]) * double(q) -
           double(orc_f16_to_f32(dmin_bits)) * double(m[j]);
}

void orc_dequant_q4_k(const uint8_t* W, int N, int K, double* w_out) {
    for (int n = 0; n < N; ++n)
        for (int k = 0; k < K; ++k) w_out[int64_t(n) * K + k] = q4_k_weight(W, K, n, k);
}

// y[m][n] = sum_k w[n][k] * x[m][k] (x is M x K, FP32), summed in f64; T = sum |w * x|.
void orc_gemv_q4_k(int M, int N, int K, const float* x, const uint8_t* W, double* y, double* T, int nthreads) {
    auto one = [&](int64_t e) {
        const int m = int(e / N), n = int(e % N);
        double acc = 0.0, tabs = 0.0;
        for (int k = 0; k < K; ++k) {
            const double t = q4_k_weight(W, K, n, k) * double(x[int64_t(m) * K + k]);
            acc += t;
            tabs += std::fabs(t);
        }
        y[e] = acc;
        if (T) T[e] = tabs;
    };
    parallel_over(int64_t(M) * N, nthreads, one);
}

// Input gradient, "Backward Pass: Gradient w.r.t. Input": dX[m][k] = sum_n w[n][k] *
// dY[m][n] (dY is M x N), summed in f64; T = sum |w * dY|. The weights get no gradient.
void orc_gemv_q4_k_backward(int M, int N, int K, const float* dY, const uint8_t* W, double* dX, double* T,
                            int nthreads) {
    auto one = [&](int64_t e) {
        const int m = int(e / K), k = int(e % K);
        double acc = 0.0, tabs = 0.0;
        for (int n = 0; n < N; ++n) {
            const double t = q4_k_weight(W, K, n, k) * double(dY[int64_t(m) * N + n]);
            acc += t;
            tabs += std::fabs(t);
        }
        dX[e] = acc;
        if (T) T[e] = tabs;
    };
    parallel_over(int64_t(M) * K, nthreads, one);
}

}  // extern "C"
