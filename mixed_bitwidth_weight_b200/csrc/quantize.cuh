// Quantiser: fp16 weights W [K][N] (act-order rows) and the block widths ->
// codes [K][N] and one fp16 scale per (128-row group, column), the step
// before qgemm_pack.
//
// The method (nightvoyager.top exllamav2 report, "关键设计决策", the adaptive
// scale paragraph): each group scale is quantised to 4 bits against the
// column's largest, qs = rint(sqrt(base / qmax) * 16), and the layer scans 96
// candidate factors p of the scales, keeping the one with the lowest squared
// error.  The group base is the largest |w| / 2^(b-1) over the group's blocks
// (the smallest scale at which no weight exceeds its block's largest code
// magnitude); p_i = (32 + i) / 96, i = 0..95; s = fp16(p (qmax qs^2 / 256));
// q = clamp(rint(w (1 / s)) + 2^(b-1), 0, 2^b - 1); the error of a candidate
// is the sum over columns (in order) of the sum over rows (in order) of
// (w - (q - 2^(b-1)) s)^2 in double; the lowest index wins a tie.
//
// Codes are decided in single precision with every operation rounded to
// nearest even (the __f*_rn intrinsics: no contraction), errors in double
// (__d*_rn), so the results are the same bits on every run and match any
// implementation that follows the same order of operations.
//
// Three kernels, all bounded by reading W (2 bytes per weight per pass):
//   quant_scan_kernel   one thread per column: pass 1 finds the group bases
//                       and qmax, pass 2 stages each group's 128 x 64 tile in
//                       shared memory and evaluates all 96 candidates on it,
//                       each candidate's running error in shared memory;
//                       writes the [96][N] column errors;
//   quant_pick_kernel   one thread per candidate sums its column errors in
//                       column order; thread 0 picks the smallest;
//   quant_emit_kernel   one thread per column writes the chosen codes and
//                       scales.
#pragma once

#include "common.cuh"

namespace qg {

constexpr int kQuantCands = 96;
constexpr int kQuantCols = 64;  // columns (threads) per scan CTA

struct QuantParams {
    const __half* w;     // [K][N]
    const uint8_t* bits; // [K/32]
    float* base;         // [G][N] workspace
    float* qmax;         // [N] workspace
    double* colerr;      // [96][N] workspace
    double* err;         // [96] out (workspace if the caller passes none)
    int32_t* best;       // [1] out (workspace if the caller passes none)
    uint8_t* codes;      // [K][N]
    __half* scales;      // [G][N]
    int K, N, G;
};

QG_DEV float quant_factor(int i) { return __fdiv_rn((float)(32 + i), 96.0f); }

// 4-bit second-level scale of a group (as a float 1..16).
QG_DEV float quant_qs(float base, float qmax) {
    if (qmax == 0.f) return 16.f;
    const float t = rintf(__fmul_rn(__fsqrt_rn(__fdiv_rn(base, qmax)), 16.f));
    return fminf(fmaxf(t, 1.f), 16.f);
}

QG_DEV __half quant_scale(float p, float qmax, float qs) {
    const float u = __fmul_rn(qmax, __fdiv_rn(__fmul_rn(qs, qs), 256.f));  // qs^2 and /256 exact
    return __float2half_rn(__fmul_rn(p, u));
}

// Code of one weight under scale s (inv = 1 / s); the zero point where s is 0.
QG_DEV int quant_code(float x, float s, float inv, int b) {
    const int z = 1 << (b - 1);
    if (s == 0.f) return z;
    float t = rintf(__fmul_rn(x, inv));
    if (t != t) t = 0.f;  // not a number: the zero point
    t = fminf(fmaxf(t, (float)(-z)), (float)((1 << b) - 1 - z));
    return (int)t + z;
}

QG_DEV double quant_err(float x, int q, int b, float s) {
    const float r = __fmul_rn((float)(q - (1 << (b - 1))), s);  // exact
    const double d = __dsub_rn((double)x, (double)r);
    return __dmul_rn(d, d);
}

// Largest |w| / 2^(b-1) of each group of column n, and their maximum.
QG_DEV float quant_bases(const QuantParams& p, int n, const uint8_t* s_bits) {
    float qmax = 0.f;
    for (int g = 0; g < p.G; ++g) {
        float base = 0.f;
        const int k1 = min(p.K, (g + 1) * 128);
        for (int k = g * 128; k < k1; ++k) {
            const float a = fabsf(__half2float(p.w[(size_t)k * p.N + n]));
            const float r = __fmul_rn(a, __int_as_float((128 - s_bits[k >> 5]) << 23));  // / 2^(b-1), exact
            base = fmaxf(base, r);
        }
        p.base[(size_t)g * p.N + n] = base;
        qmax = fmaxf(qmax, base);
    }
    return qmax;
}

__global__ void __launch_bounds__(kQuantCols) quant_scan_kernel(const QuantParams p) {
    extern __shared__ __align__(1024) uint8_t smem[];  // one alignment for every kernel of the library
    double* s_acc = reinterpret_cast<double*>(smem);                          // [96][kQuantCols]
    __half* s_tile = reinterpret_cast<__half*>(s_acc + kQuantCands * kQuantCols);  // [128][kQuantCols]
    uint8_t* s_bits = reinterpret_cast<uint8_t*>(s_tile + 128 * kQuantCols);  // [K/32]
    const int t = threadIdx.x;
    const int n0 = blockIdx.x * kQuantCols;
    const int n = n0 + t;
    const bool live = n < p.N;
    for (int j = t; j < p.K / 32; j += kQuantCols) {
        int b = p.bits[j];
        if (!width_ok(b)) {
            if (blockIdx.x == 0) set_dev_error(QGEMM_DEV_BAD_SCHEDULE);
            b = 2;  // keeps every shift below in range; the call reports the error
        }
        s_bits[j] = (uint8_t)b;
    }
    for (int i = 0; i < kQuantCands; ++i) s_acc[i * kQuantCols + t] = 0.0;
    __syncthreads();
    const float qmax = live ? quant_bases(p, n, s_bits) : 0.f;
    if (live) p.qmax[n] = qmax;
    for (int g = 0; g < p.G; ++g) {
        const int k0 = g * 128, rows = min(128, p.K - k0);
        __syncthreads();  // the previous group's tile is no longer read
        for (int e = t; e < rows * kQuantCols; e += kQuantCols) {
            const int r = e / kQuantCols, c = e - r * kQuantCols;
            s_tile[e] = (n0 + c < p.N) ? p.w[(size_t)(k0 + r) * p.N + n0 + c] : __float2half_rn(0.f);
        }
        __syncthreads();
        if (!live) continue;
        const float qs = quant_qs(p.base[(size_t)g * p.N + n], qmax);
        for (int i = 0; i < kQuantCands; ++i) {
            const float s = __half2float(quant_scale(quant_factor(i), qmax, qs));
            const float inv = (s == 0.f) ? 0.f : __fdiv_rn(1.f, s);
            double acc = s_acc[i * kQuantCols + t];
            for (int r = 0; r < rows; ++r) {
                const int b = s_bits[(k0 + r) >> 5];
                const float x = __half2float(s_tile[r * kQuantCols + t]);
                acc = __dadd_rn(acc, quant_err(x, quant_code(x, s, inv, b), b, s));
            }
            s_acc[i * kQuantCols + t] = acc;
        }
    }
    if (live)
        for (int i = 0; i < kQuantCands; ++i) p.colerr[(size_t)i * p.N + n] = s_acc[i * kQuantCols + t];
}

__global__ void __launch_bounds__(kQuantCands) quant_pick_kernel(const QuantParams p) {
    __shared__ double s_e[kQuantCands];
    const int i = threadIdx.x;
    double e = 0.0;
    for (int n = 0; n < p.N; ++n) e = __dadd_rn(e, p.colerr[(size_t)i * p.N + n]);
    s_e[i] = e;
    p.err[i] = e;
    __syncthreads();
    if (i == 0) {
        int best = 0;
        for (int c = 1; c < kQuantCands; ++c)
            if (s_e[c] < s_e[best]) best = c;
        *p.best = best;
    }
}

__global__ void __launch_bounds__(128) quant_emit_kernel(const QuantParams p) {
    const int n = blockIdx.x * 128 + threadIdx.x;
    if (n >= p.N) return;
    const float pf = quant_factor(*p.best);
    const float qmax = p.qmax[n];
    for (int g = 0; g < p.G; ++g) {
        const __half sh = quant_scale(pf, qmax, quant_qs(p.base[(size_t)g * p.N + n], qmax));
        p.scales[(size_t)g * p.N + n] = sh;
        const float s = __half2float(sh);
        const float inv = (s == 0.f) ? 0.f : __fdiv_rn(1.f, s);
        const int k1 = min(p.K, (g + 1) * 128);
        for (int k = g * 128; k < k1; ++k) {
            const int b = width_ok(p.bits[k >> 5]) ? p.bits[k >> 5] : 2;
            p.codes[(size_t)k * p.N + n] =
                (uint8_t)quant_code(__half2float(p.w[(size_t)k * p.N + n]), s, inv, b);
        }
    }
}

}  // namespace qg
