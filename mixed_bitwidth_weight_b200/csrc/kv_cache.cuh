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
// One warp per vector; lane l holds E = D/32 consecutive elements (vector
// loads and stores), so a group of 32 elements is 32/E consecutive lanes and
// its largest magnitude takes log2(32/E) shuffles.  The groups' code streams
// follow one another, so lane l's E codes are bits [E b l, E b (l + 1)) of the
// vector's stream, and lane j assembles word j from the two to four lanes
// whose bits it holds, one coalesced store per lane.  The
// fast Walsh-Hadamard transform runs in single precision in the order strides
// 1, 2, ..., D/2, each stage replacing (a at i, b at i + stride) by
// (a + b, a - b): strides below E pair a lane's registers, larger ones pair
// lanes.  Every operation rounds to
// nearest even, so the codes are the same bits as any implementation of the
// same steps.  Both kernels read and write each byte once (HBM-bound).
#pragma once

#include "common.cuh"

namespace qg {

constexpr int kKvWarps = 8;  // vectors per CTA (one per warp)

// Fast Walsh-Hadamard transform of one vector held by a warp, E = D / 32
// consecutive elements per lane (lane l holds elements E l .. E l + E - 1):
// strides below E pair registers of a lane, larger strides pair lanes
// (shuffles); the stages run in stride order 1, 2, 4, ...
template <int E>
QG_DEV void fwht_warp(float (&x)[E], int lane) {
#pragma unroll
    for (int st = 1; st < E; st <<= 1)
#pragma unroll
        for (int i = 0; i < E; ++i)
            if (!(i & st)) {
                const float a = x[i], c = x[i + st];
                x[i] = __fadd_rn(a, c);
                x[i + st] = __fsub_rn(a, c);
            }
#pragma unroll
    for (int ls = 1; ls < 32; ls <<= 1) {  // element stride E * ls
        const bool hi = (lane & ls) != 0;
#pragma unroll
        for (int i = 0; i < E; ++i) {
            const float o = __shfl_xor_sync(0xffffffffu, x[i], ls);
            x[i] = hi ? __fsub_rn(o, x[i]) : __fadd_rn(x[i], o);
        }
    }
}

// Groups of 32 elements are 32 / E consecutive lanes; lane-in-group g = lane % (32 / E).
// b = B bits per code.
template <int E, int B>
__global__ void __launch_bounds__(32 * kKvWarps) kv_quant_kernel(const __half* __restrict__ v, int64_t nvec,
                                                                uint32_t* __restrict__ codes,
                                                                __half* __restrict__ scales) {
    constexpr int D = 32 * E, G = 32 / E;  // lanes per group
    constexpr int b = B;
    const int lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * kKvWarps + (threadIdx.x >> 5);
    if (t >= nvec) return;  // whole warps only
    float x[E];
    const __half* src = v + t * D + E * lane;
    if constexpr (E == 1) {
        x[0] = __half2float(src[0]);
    } else if constexpr (E == 2) {
        const __half2 h = *reinterpret_cast<const __half2*>(src);
        x[0] = __low2float(h);
        x[1] = __high2float(h);
    } else {
#pragma unroll
        for (int i = 0; i < E; i += 4) {
            const uint2 u = *reinterpret_cast<const uint2*>(src + i);
            x[i] = __low2float(*reinterpret_cast<const __half2*>(&u.x));
            x[i + 1] = __high2float(*reinterpret_cast<const __half2*>(&u.x));
            x[i + 2] = __low2float(*reinterpret_cast<const __half2*>(&u.y));
            x[i + 3] = __high2float(*reinterpret_cast<const __half2*>(&u.y));
        }
    }
    fwht_warp<E>(x, lane);
    constexpr int z = 1 << (b - 1);
    const int grp = lane / G, gl = lane % G;  // group of this lane, lane within it
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < E; ++i) amax = fmaxf(amax, fabsf(x[i]));
#pragma unroll
    for (int o = 1; o < G; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const __half sh = __float2half_rn(__fdiv_rn(amax, (float)(z - 1)));
    const float s = __half2float(sh);
    const float inv = (s == 0.f) ? 0.f : __frcp_rn(s);  // the correctly rounded 1 / s
    // this lane's E codes: bits [c l, c l + c) of the vector's stream, c = E b
    // (group g's b words follow group g - 1's, so the groups' streams join)
    uint64_t chunk = 0;
#pragma unroll
    for (int i = 0; i < E; ++i) {
        int q = z;
        if (s != 0.f) {
            float tq = rintf(__fmul_rn(x[i], inv));
            if (tq != tq) tq = 0.f;  // not a number: the zero point
            tq = fminf(fmaxf(tq, (float)(-z)), (float)(z - 1));
            q = (int)tq + z;
        }
        chunk |= (uint64_t)q << (i * b);
    }
    // word j of the c words: the chunks of lanes floor(32 j / c) ..
    // floor((32 j + 31) / c), at most floor(31 / c) + 2 of them; lane j
    // gathers word j (and j + 32 when c > 32)
    constexpr int c = E * b;
    constexpr int nsrc = 31 / c + 2;
    const uint32_t clo = (uint32_t)chunk, chi = (uint32_t)(chunk >> 32);
    uint32_t* wv = codes + t * c;
#pragma unroll
    for (int pass = 0; pass < (E == 8 ? 2 : 1); ++pass) {
        const int j = lane + 32 * pass;
        const int l0 = (32 * j) / c, l1 = (32 * j + 31) / c;
        uint32_t word = 0;
#pragma unroll
        for (int r = 0; r < nsrc; ++r) {
            const int l = min(l0 + r, 31);
            const uint32_t vlo = __shfl_sync(0xffffffffu, clo, l);
            const uint32_t vhi = (E * 8 > 32) ? __shfl_sync(0xffffffffu, chi, l) : 0u;
            const uint64_t v = ((uint64_t)vhi << 32) | vlo;
            const int d = c * l - 32 * j;  // the chunk's first bit relative to the word
            if (l0 + r <= l1) word |= (d >= 0) ? (uint32_t)(v << d) : (uint32_t)(v >> (-d));
        }
        if (j < c) wv[j] = word;
    }
    if (gl == 0) scales[t * E + grp] = sh;
}

template <int E>
__global__ void __launch_bounds__(32 * kKvWarps) kv_dequant_kernel(const uint32_t* __restrict__ codes,
                                                                  const __half* __restrict__ scales, int64_t nvec,
                                                                  int b, __half* __restrict__ v) {
    constexpr int D = 32 * E, G = 32 / E;
    const int lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * kKvWarps + (threadIdx.x >> 5);
    if (t >= nvec) return;
    const int z = 1 << (b - 1);
    const int grp = lane / G, gl = lane % G;
    const uint32_t* w = codes + (t * E + grp) * b;
    const int pos = E * gl * b, wi = pos >> 5, o = pos & 31;
    // the chunk spans at most three words (E b <= 64 bits)
    const uint64_t lo = w[wi] | ((wi + 1 < b) ? (uint64_t)w[wi + 1] << 32 : 0ull);
    uint64_t chunk = lo >> o;
    if (o > 0 && wi + 2 < b) chunk |= (uint64_t)w[wi + 2] << (64 - o);
    const float s = __half2float(scales[t * E + grp]);
    const uint64_t mask = (1ull << b) - 1ull;
    float x[E];
#pragma unroll
    for (int i = 0; i < E; ++i) x[i] = __fmul_rn((float)((int)((chunk >> (i * b)) & mask) - z), s);  // exact
    fwht_warp<E>(x, lane);
    __half* dst = v + t * D + E * lane;
    const float inv_d = 1.f / (float)D;  // a power of two: exact
    if constexpr (E == 1) {
        dst[0] = __float2half_rn(__fmul_rn(x[0], inv_d));
    } else {
#pragma unroll
        for (int i = 0; i < E; i += 2)
            *reinterpret_cast<__half2*>(dst + i) =
                __floats2half2_rn(__fmul_rn(x[i], inv_d), __fmul_rn(x[i + 1], inv_d));
    }
}

}  // namespace qg
