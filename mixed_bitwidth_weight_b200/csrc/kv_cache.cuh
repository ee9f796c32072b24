// KV-cache quantisation with a Hadamard rotation: fp16 (token, head) vectors
// of length D <-> b-bit codes with one fp16 scale per 32 elements
// (nightvoyager.top exllamav2 report, "创新之处": K/V are rotated by a
// Hadamard matrix and then quantised to 4 bits, the rotation spreading
// outlier channels over the whole vector; navi2ai ExLlamaV3 page, "核心能力":
// 2-8 bit caches).
//
// Quantise:   u = H_D v (Sylvester matrix, no normalisation), per group of 32
//             s = fp16(max|u| / (2^(b-1) - 1)),
//             q = clamp(rint(u (1 / s)) + 2^(b-1), 0, 2^b - 1) (the zero point
//             where s is 0), packed like the weights' 32-code blocks: b words,
//             code r at bits [r b, r b + b) of the LSB-first stream.
// Dequantise: u' = (q - 2^(b-1)) s, v' = fp16((H_D u') / D)  (H_D H_D = D I).
//
// Each warp takes kKvPerWarp consecutive vectors and issues all their loads
// before any arithmetic; lane l holds elements l + 32 r, r = 0 .. D/32 - 1, so
// group r is register r across the warp.  The fast Walsh-Hadamard transform
// runs in single precision in the order strides 1, 2, ..., D/2, each stage
// replacing (a at i, b at i + stride) by (a + b, a - b): strides below 32 pair
// lanes (shuffles), larger strides pair registers.  Every operation rounds to
// nearest even, so the codes are the same bits as any implementation of the
// same steps.  Both kernels read and write each byte once (HBM-bound).
#pragma once

#include "common.cuh"

namespace qg {

constexpr int kKvWarps = 8;    // warps per CTA
constexpr int kKvPerWarp = 1;  // vectors per warp (measured: four per warp, loads first, was slower)

template <int R>
QG_DEV void fwht_warp(float (&x)[R], int lane) {
#pragma unroll
    for (int st = 1; st < 32; st <<= 1) {
        const bool hi = (lane & st) != 0;
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const float o = __shfl_xor_sync(0xffffffffu, x[r], st);
            x[r] = hi ? __fsub_rn(o, x[r]) : __fadd_rn(x[r], o);
        }
    }
#pragma unroll
    for (int sr = 1; sr < R; sr <<= 1)
#pragma unroll
        for (int r = 0; r < R; ++r)
            if (!(r & sr)) {
                const float a = x[r], c = x[r + sr];
                x[r] = __fadd_rn(a, c);
                x[r + sr] = __fsub_rn(a, c);
            }
}

template <int R>
__global__ void __launch_bounds__(32 * kKvWarps) kv_quant_kernel(const __half* __restrict__ v, int64_t nvec, int b,
                                                                uint32_t* __restrict__ codes,
                                                                __half* __restrict__ scales) {
    constexpr int D = 32 * R;
    const int lane = threadIdx.x & 31;
    const int64_t t0 = ((int64_t)blockIdx.x * kKvWarps + (threadIdx.x >> 5)) * kKvPerWarp;
    if (t0 >= nvec) return;  // whole warps only
    const int nv = (nvec - t0 < kKvPerWarp) ? (int)(nvec - t0) : kKvPerWarp;
    // every load of the warp's vectors first, then the arithmetic
    float x[kKvPerWarp][R];
#pragma unroll
    for (int j = 0; j < kKvPerWarp; ++j)
#pragma unroll
        for (int r = 0; r < R; ++r) x[j][r] = (j < nv) ? __half2float(v[(t0 + j) * D + 32 * r + lane]) : 0.f;
    const int z = 1 << (b - 1);
#pragma unroll
    for (int j = 0; j < kKvPerWarp; ++j) {
        if (j >= nv) break;  // uniform over the warp
        const int64_t t = t0 + j;
        fwht_warp<R>(x[j], lane);
#pragma unroll
        for (int r = 0; r < R; ++r) {
            float amax = fabsf(x[j][r]);
#pragma unroll
            for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            const __half sh = __float2half_rn(__fdiv_rn(amax, (float)(z - 1)));
            const float s = __half2float(sh);
            int q = z;
            if (s != 0.f) {
                float tq = rintf(__fmul_rn(x[j][r], __fdiv_rn(1.f, s)));
                if (tq != tq) tq = 0.f;  // not a number: the zero point
                tq = fminf(fmaxf(tq, (float)(-z)), (float)(z - 1));
                q = (int)tq + z;
            }
            uint32_t* w = codes + (t * R + r) * b;
            uint32_t mine = 0;  // lane k keeps word k
            for (int k = 0; k < b; ++k) {
                const int d = lane * b - 32 * k;  // the code's first bit, relative to word k
                uint32_t part = 0;
                if (d >= 0 && d < 32) part = (uint32_t)q << d;
                else if (d < 0 && d + b > 0) part = (uint32_t)q >> (-d);
                part = __reduce_or_sync(0xffffffffu, part);
                if (lane == k) mine = part;
            }
            if (lane < b) w[lane] = mine;
            if (lane == 0) scales[t * R + r] = sh;
        }
    }
}

template <int R>
__global__ void __launch_bounds__(32 * kKvWarps) kv_dequant_kernel(const uint32_t* __restrict__ codes,
                                                                  const __half* __restrict__ scales, int64_t nvec,
                                                                  int b, __half* __restrict__ v) {
    constexpr int D = 32 * R;
    const int lane = threadIdx.x & 31;
    const int64_t t0 = ((int64_t)blockIdx.x * kKvWarps + (threadIdx.x >> 5)) * kKvPerWarp;
    if (t0 >= nvec) return;
    const int nv = (nvec - t0 < kKvPerWarp) ? (int)(nvec - t0) : kKvPerWarp;
    const int z = 1 << (b - 1);
    const uint32_t mask = (1u << b) - 1u;
    const int p = lane * b, wi = p >> 5, o = p & 31;
    const bool two = o + b > 32;  // the code straddles two words
    // every load of the warp's vectors first (the words holding this lane's
    // codes and the group scales), then the arithmetic
    uint32_t lo[kKvPerWarp][R], hi[kKvPerWarp][R];
    float sc[kKvPerWarp][R];
#pragma unroll
    for (int j = 0; j < kKvPerWarp; ++j)
#pragma unroll
        for (int r = 0; r < R; ++r) {
            lo[j][r] = hi[j][r] = 0u;
            sc[j][r] = 0.f;
            if (j < nv) {
                const uint32_t* w = codes + ((t0 + j) * R + r) * b;
                lo[j][r] = w[wi];
                if (two) hi[j][r] = w[wi + 1];
                sc[j][r] = __half2float(scales[(t0 + j) * R + r]);
            }
        }
#pragma unroll
    for (int j = 0; j < kKvPerWarp; ++j) {
        if (j >= nv) break;  // uniform over the warp
        float x[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            uint32_t q = lo[j][r] >> o;
            if (two) q |= hi[j][r] << (32 - o);
            q &= mask;
            x[r] = __fmul_rn((float)((int)q - z), sc[j][r]);  // exact
        }
        fwht_warp<R>(x, lane);
#pragma unroll
        for (int r = 0; r < R; ++r)
            v[(t0 + j) * D + 32 * r + lane] = __float2half_rn(__fmul_rn(x[r], 1.f / (float)D));
    }
}

}  // namespace qg
