// Split-K GEMV for decode (M <= 16): y = x[:, perm] . dequant(Wq).
//
// The pages describe the decode Q-GEMM as bound by memory bandwidth: tokens are
// generated "as fast as memory bandwidth allows" with a kernel "near the
// memory-bandwidth limit" (navi2ai ExLlamaV3 page, "项目概述" and "核心能力").
// This kernel is built to stream the packed words at HBM speed on B200.
//
// Work split.  W is cut into 256-column tiles; a unit is (tile t, 32-row block
// j) and costs b_j packed word rows.  Units are ordered tile-major and the
// sequence is cut into gridDim.x contiguous ranges of equal word-row cost, one
// per CTA (grid = number of SMs), so every SM streams the same number of bytes
// whatever the width mix.  A tile covered by several CTAs is reduced by the
// last of them to finish (an atomic ticket, no waiting): partial sums go to a
// workspace slot and the last CTA adds the slots in CTA order (deterministic).
//
// Inside a CTA.  Warp 8 is the producer: one lane streams the word rows of each
// unit (and, at the start of each 128-row group, the scale row) with
// cp.async.bulk into a ring of shared-memory rows and signals a per-unit
// "full" mbarrier.  Warps 0-7 are consumers, 32 columns each.  For every unit a
// consumer lane decodes 8 codes for each of its columns straight into fp16
// (code - zero) pairs with the lop3/prmt "magic exponent" trick and feeds them
// as the A operand of mma.sync m16n8k16 (A = W^T: 16 output columns x 16 k),
// with the staged activations as B (16 k x 8 tokens).  The MMA cost per weight
// is the same for M = 1 and M = 8, so decode stays bound by the word stream.
// The scale is applied once per (group, column) to an fp32 group accumulator.
//
// Activations are gathered once per CTA through perm into shared memory, in
// the order in which each block width's decoder emits codes.
#pragma once

#include "pack_dequant.cuh"

namespace qg {

constexpr int kGemvTileCols = 256;
constexpr int kGemvConsumerWarps = 8;
constexpr int kGemvConsumers = kGemvConsumerWarps * 32;
constexpr int kGemvThreads = kGemvConsumers + 32;
constexpr int kGemvRowWords = kGemvTileCols + 8;  // +8 words: rotates banks by 8 per row
constexpr int kGemvRowBytes = kGemvRowWords * 4;
constexpr int kGemvSlots = 64;                    // units in flight (mbarrier pairs)
constexpr int kGemvMaxRing = 192;                 // ring rows (cap)
constexpr int kGemvMinRing = 24;
constexpr int kGemvMaxCtas = 1024;
constexpr int kGemvSmemBudget = 227 * 1024;

struct GemvParams {
    const void* x;
    const int32_t* perm;
    const uint32_t* qw;
    int64_t qw_rows;
    const __half* scales;
    const uint8_t* bits;
    const int32_t* offs;
    __half* y;
    int* tickets;   // [tiles]
    float* slots;   // [gridDim.x][2][MP][256]
    int M, K, N, nb, tiles;
    int x_bf16;
    int ring_rows;  // rows in the shared-memory ring
    int span_cap;   // blocks the activation stage can hold
};

// fp16 bit pattern of num / 2^log2_den for values exactly representable as
// normal fp16 numbers (only used for the decoder's constants).
constexpr uint32_t f16_exact(int num, int log2_den) {
    uint32_t sign = num < 0 ? 0x8000u : 0u;
    uint32_t a = (uint32_t)(num < 0 ? -num : num);
    int e = 0;
    while (a < 1024u) { a <<= 1; --e; }
    while (a >= 2048u) { a >>= 1; ++e; }
    return sign | ((uint32_t)(e - log2_den + 25) << 10) | (a - 1024u);
}
constexpr uint32_t h2(int num, int log2_den) {
    return f16_exact(num, log2_den) * 0x10001u;
}
constexpr uint32_t kMagic = 0x64006400u;  // fp16x2 {1024, 1024}

// Code index (0..31 within the block) held at stage position pos = c*8 + p*2 + h:
// lane quad c, pair p of the lane's four fp16x2 registers, half h.  This is the
// order in which decode<B> below emits codes; activations are staged in the
// same order so that A and B of each mma.sync agree on k.
QG_DEV int code_of_pos(int b, int pos) {
    const int c = pos >> 3, p = (pos >> 1) & 3, h = pos & 1;
    if (b == 2) return 16 * (c >> 1) + 4 * (c & 1) + p + 8 * h;
    if (b == 8) return (p < 2) ? (4 * c + p + 2 * h) : (16 + 4 * c + (p - 2) + 2 * h);
    return 8 * c + p + 4 * h;  // b = 3, 4, 5, 6
}

// Address of word i of the current unit for column col in the ring.
QG_DEV const uint32_t* ring_word(const uint8_t* ring, int R, int row, int col) {
    if (row >= R) row -= R;
    return reinterpret_cast<const uint32_t*>(ring + (size_t)row * kGemvRowBytes) + col;
}

// Decode the 8 codes lane quad c owns in one column into four fp16x2 values
// (q - 2^(B-1)), exact.  (h & mask) | 0x6400 is the fp16 number 1024 + q*2^P
// for a code at mantissa bits [P, P+B); one fma by 2^-P and -(2^(10-P) + zero)
// turns it into q - zero exactly.
template <int B>
QG_DEV void decode(const uint8_t* ring, int R, int base, int col, int c, uint32_t (&P)[4]) {
    if constexpr (B == 2) {
        uint32_t v = *ring_word(ring, R, base + (c >> 1), col);
        v >>= (c & 1) * 8;
        P[0] = hfma2_u32(lop3_and_or(v, 0x00030003u, kMagic), h2(1, 0), h2(-1026, 0));
        P[1] = hfma2_u32(lop3_and_or(v, 0x000C000Cu, kMagic), h2(1, 2), h2(-258, 0));
        P[2] = hfma2_u32(lop3_and_or(v, 0x00300030u, kMagic), h2(1, 4), h2(-66, 0));
        P[3] = hfma2_u32(lop3_and_or(v, 0x00C000C0u, kMagic), h2(1, 6), h2(-18, 0));
    } else if constexpr (B == 3) {
        const int lo = (c <= 1) ? 0 : c - 1;
        const int hi = (c <= 1) ? 1 : 2;
        const int s0 = (c == 0) ? 0 : 32 - 8 * c;  // 0, 24, 16, 8
        const uint32_t wl = *ring_word(ring, R, base + lo, col);
        const uint32_t wh = *ring_word(ring, R, base + hi, col);
        const uint32_t X = __funnelshift_r(wl, wh, s0);       // codes i at bits 3i
        const uint32_t u = (X & 0xFFFFu) | ((X << 4) & 0xFFFF0000u);
        P[0] = hfma2_u32(lop3_and_or(u, 0x00070007u, kMagic), h2(1, 0), h2(-1028, 0));
        P[1] = hfma2_u32(lop3_and_or(u, 0x00380038u, kMagic), h2(1, 3), h2(-132, 0));
        P[2] = hfma2_u32(lop3_and_or(u, 0x01C001C0u, kMagic), h2(1, 6), h2(-20, 0));
        P[3] = hfma2_u32(lop3_and_or(u >> 9, 0x00070007u, kMagic), h2(1, 0), h2(-1028, 0));
    } else if constexpr (B == 4) {
        const uint32_t v = *ring_word(ring, R, base + c, col);
        const uint32_t v2 = v >> 8;
        P[0] = hfma2_u32(lop3_and_or(v, 0x000F000Fu, kMagic), h2(1, 0), h2(-1032, 0));
        P[1] = hfma2_u32(lop3_and_or(v, 0x00F000F0u, kMagic), h2(1, 4), h2(-72, 0));
        P[2] = hfma2_u32(lop3_and_or(v2, 0x000F000Fu, kMagic), h2(1, 0), h2(-1032, 0));
        P[3] = hfma2_u32(lop3_and_or(v2, 0x00F000F0u, kMagic), h2(1, 4), h2(-72, 0));
    } else if constexpr (B == 5) {
        const int lo = c;                 // floor(40c / 32) = c for c < 4
        const int s0 = (8 * c) & 31;      // 40c mod 32
        const uint32_t wl = *ring_word(ring, R, base + lo, col);
        const uint32_t wh = *ring_word(ring, R, base + lo + 1, col);
        const uint64_t X = (((uint64_t)wh << 32) | wl) >> s0;  // codes i at bits 5i
        const uint32_t u1 = prmt((uint32_t)X, (uint32_t)(X >> 20), 0x5410);
        const uint32_t u2 = prmt((uint32_t)(X >> 10), (uint32_t)(X >> 30), 0x5410);
        P[0] = hfma2_u32(lop3_and_or(u1, 0x001F001Fu, kMagic), h2(1, 0), h2(-1040, 0));
        P[1] = hfma2_u32(lop3_and_or(u1, 0x03E003E0u, kMagic), h2(1, 5), h2(-48, 0));
        P[2] = hfma2_u32(lop3_and_or(u2, 0x001F001Fu, kMagic), h2(1, 0), h2(-1040, 0));
        P[3] = hfma2_u32(lop3_and_or(u2, 0x03E003E0u, kMagic), h2(1, 5), h2(-48, 0));
    } else if constexpr (B == 6) {
        const int lo = (c < 2) ? c : c + 1;  // 0, 1, 3, 4
        const int s0 = (c & 1) * 16;         // 0, 16, 0, 16
        const uint32_t wl = *ring_word(ring, R, base + lo, col);
        const uint32_t wh = *ring_word(ring, R, base + lo + 1, col);
        const uint64_t X = (((uint64_t)wh << 32) | wl) >> s0;  // codes i at bits 6i
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t u = prmt((uint32_t)(X >> (6 * i)), (uint32_t)(X >> (6 * i + 24)), 0x5410);
            P[i] = hfma2_u32(lop3_and_or(u, 0x003F003Fu, kMagic), h2(1, 0), h2(-1056, 0));
        }
    } else {  // B == 8
        const uint32_t v0 = *ring_word(ring, R, base + c, col);
        const uint32_t v1 = *ring_word(ring, R, base + c + 4, col);
        P[0] = hfma2_u32(prmt(v0, 0x64646464u, 0x4240), h2(1, 0), h2(-1152, 0));
        P[1] = hfma2_u32(prmt(v0, 0x64646464u, 0x4341), h2(1, 0), h2(-1152, 0));
        P[2] = hfma2_u32(prmt(v1, 0x64646464u, 0x4240), h2(1, 0), h2(-1152, 0));
        P[3] = hfma2_u32(prmt(v1, 0x64646464u, 0x4341), h2(1, 0), h2(-1152, 0));
    }
}

template <int B, int MT>
QG_DEV void unit_mma(const uint8_t* ring, int R, int base, int colw, int g, int c,
                     const uint4 (&xf)[MT], float (&acc)[MT][2][4]) {
#pragma unroll
    for (int cg = 0; cg < 2; ++cg) {
        uint32_t P[4], Q[4];
        decode<B>(ring, R, base, colw + cg * 16 + g, c, P);
        decode<B>(ring, R, base, colw + cg * 16 + g + 8, c, Q);
#pragma unroll
        for (int ts = 0; ts < MT; ++ts) {
            mma_f16_16816(acc[ts][cg], P[0], Q[0], P[1], Q[1], xf[ts].x, xf[ts].y);
            mma_f16_16816(acc[ts][cg], P[2], Q[2], P[3], Q[3], xf[ts].z, xf[ts].w);
        }
    }
}

// First unit of CTA i: the first unit whose cost prefix reaches ceil(i*C/G).
QG_DEV int64_t unit_start(int64_t i, int64_t G, int64_t C, int64_t W, int nb, int tiles,
                          const int32_t* s_offs) {
    if (i >= G) return (int64_t)tiles * nb;
    const int64_t pos = (i * C + G - 1) / G;
    int64_t t = pos / W;
    const int64_t rem = pos - t * W;
    int lo = 0, hi = nb;  // first j in [0, nb] with offs[j] >= rem
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (s_offs[mid] >= rem) hi = mid; else lo = mid + 1;
    }
    int64_t u = t * nb + lo;  // lo == nb rolls over to the next tile's block 0
    return u;
}

// CTA that owns unit u.
QG_DEV int cta_of(int64_t u, int64_t G, int64_t C, int64_t W, int nb, const int32_t* s_offs) {
    const int64_t t = u / nb;
    const int j = (int)(u - t * nb);
    const int64_t pos = t * W + s_offs[j];
    return (int)((pos * G) / C);
}

template <int MT>
__global__ void __launch_bounds__(kGemvThreads, 1) gemv_kernel(const GemvParams p) {
    constexpr int MP = MT * 8;
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nb = p.nb;

    int32_t* s_offs = reinterpret_cast<int32_t*>(smem);
    size_t o = ((size_t)(nb + 1) * 4 + 15) & ~(size_t)15;
    uint64_t* s_full = reinterpret_cast<uint64_t*>(smem + o);
    o += kGemvSlots * 8;
    uint64_t* s_empty = reinterpret_cast<uint64_t*>(smem + o);
    o += kGemvSlots * 8;
    int* s_misc = reinterpret_cast<int*>(smem + o);  // bad schedule, last flag, abort
    int* s_emax = s_misc + 16;                       // per-row largest bf16 exponent field
    o += 128;
    __half* s_x = reinterpret_cast<__half*>(smem + o);
    o += ((size_t)p.span_cap * p.M * 64 + 15) & ~(size_t)15;
    uint8_t* s_ring = smem + o;
    const int R = p.ring_rows;

    // ---- schedule into shared memory, validated before any weight access
    if (tid < 32) s_misc[tid] = 0;
    for (int i = tid; i <= nb; i += kGemvThreads) s_offs[i] = p.offs[i];
    __syncthreads();
    bool bad = false;
    for (int j = tid; j < nb; j += kGemvThreads) {
        const int b = p.bits[j];
        if (!width_ok(b) || s_offs[j + 1] - s_offs[j] != b) bad = true;
    }
    if (tid == 0 && (s_offs[0] != 0 || (int64_t)s_offs[nb] != p.qw_rows)) bad = true;
    if (bad) atomicOr(&s_misc[0], 1);
    if (tid == 0) {
        for (int i = 0; i < kGemvSlots; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&s_empty[i], kGemvConsumerWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();
    if (s_misc[0]) {
        if (tid == 0) set_dev_error(QGEMM_DEV_BAD_SCHEDULE);
        return;
    }

    const int64_t W = s_offs[nb];
    const int64_t C = (int64_t)p.tiles * W;
    const int64_t G = gridDim.x;
    const int64_t u0 = unit_start(blockIdx.x, G, C, W, nb, p.tiles, s_offs);
    const int64_t u1 = unit_start(blockIdx.x + 1, G, C, W, nb, p.tiles, s_offs);
    const int64_t nunits = u1 - u0;
    if (nunits <= 0) return;

    // =================================================== producer warp
    if (warp == kGemvConsumerWarps) {
        if (lane != 0) return;
        const uint64_t policy = policy_evict_first();
        int t = (int)(u0 / nb), j = (int)(u0 - (int64_t)t * nb);
        int jr = j;
        int64_t rows_issued = 0, rows_released = 0, k_rel = 0;
        int ring_row = 0;
        bool ok = true;
        int64_t k = 0;
        for (; k < nunits && ok; ++k) {
            const int b = s_offs[j + 1] - s_offs[j];
            const bool hs = ((j & 3) == 0) || (k == 0);
            const int need = b + (hs ? 1 : 0);
            while (k - k_rel >= kGemvSlots || rows_issued + need - rows_released > R) {
                if (!mbar_wait(&s_empty[k_rel % kGemvSlots], (uint32_t)((k_rel / kGemvSlots) & 1))) {
                    ok = false;
                    break;
                }
                const int br = s_offs[jr + 1] - s_offs[jr];
                rows_released += br + ((((jr & 3) == 0) || k_rel == 0) ? 1 : 0);
                ++k_rel;
                if (++jr == nb) jr = 0;
            }
            if (!ok) break;
            const int slot = (int)(k % kGemvSlots);
            const int cols = min(kGemvTileCols, p.N - t * kGemvTileCols);
            const uint32_t bytes = (uint32_t)(b * cols * 4 + (hs ? cols * 2 : 0));
            mbar_arrive_expect_tx(&s_full[slot], bytes);
            const uint32_t* src = p.qw + (size_t)s_offs[j] * p.N + (size_t)t * kGemvTileCols;
            for (int r = 0; r < b; ++r) {
                bulk_g2s_hint(s_ring + (size_t)ring_row * kGemvRowBytes, src + (size_t)r * p.N,
                              (uint32_t)cols * 4, &s_full[slot], policy);
                if (++ring_row == R) ring_row = 0;
            }
            if (hs) {
                bulk_g2s(s_ring + (size_t)ring_row * kGemvRowBytes,
                         p.scales + (size_t)(j >> 2) * p.N + (size_t)t * kGemvTileCols,
                         (uint32_t)cols * 2, &s_full[slot]);
                if (++ring_row == R) ring_row = 0;
            }
            rows_issued += need;
            if (++j == nb) { j = 0; ++t; }
        }
        if (!ok) {
            s_misc[2] = 1;
            // let copies already in flight land before the CTA can exit
            for (int64_t kk = k_rel; kk < k; ++kk)
                mbar_wait(&s_full[kk % kGemvSlots], (uint32_t)((kk / kGemvSlots) & 1));
        }
        return;
    }

    // =================================================== consumer warps
    const int ctid = tid;  // 0..255
    const int M = p.M;

    // ---- gather activations through perm into the stage, decoder order
    const int span = (int)min((int64_t)nb, nunits);
    const int j_first = (int)(u0 % nb);
    {
        const int total = span * 32;
        for (int e0 = ctid; e0 < total; e0 += kGemvConsumers * 4) {
            int src[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int e = e0 + q * kGemvConsumers;
                src[q] = 0;
                if (e < total) {
                    int jj = j_first + (e >> 5);
                    if (jj >= nb) jj -= nb;
                    const int b = s_offs[jj + 1] - s_offs[jj];
                    int s = p.perm[jj * 32 + code_of_pos(b, e & 31)];
                    if (s < 0 || s >= p.K) {
                        set_dev_error(QGEMM_DEV_BAD_PERM);
                        s = 0;
                    }
                    src[q] = s;
                }
            }
            for (int m = 0; m < M; ++m) {
                uint16_t v[4];
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    v[q] = reinterpret_cast<const uint16_t*>(p.x)[(size_t)m * p.K + src[q]];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int e = e0 + q * kGemvConsumers;
                    if (e < total) {
                        reinterpret_cast<uint16_t*>(s_x)[((size_t)(e >> 5) * M + m) * 32 + (e & 31)] = v[q];
                        if (p.x_bf16) atomicMax(&s_emax[m], (int)((v[q] >> 7) & 0xFF));
                    }
                }
            }
        }
    }
    // bf16 activations are rescaled per row by 2^-shift into fp16 range (the
    // row's largest magnitude lands in [2^14, 2^15)); outputs are multiplied
    // back by 2^shift.  fp16 activations are used as they are (shift 0).
    if (p.x_bf16) {
        named_bar_sync(1, kGemvConsumers);
        const int total = span * 32;
        for (int e = ctid; e < total; e += kGemvConsumers)
            for (int m = 0; m < M; ++m) {
                const int shift = s_emax[m] == 0 ? 0 : s_emax[m] - 141;
                const float in1 = __int_as_float((127 - shift / 2) << 23);
                const float in2 = __int_as_float((127 - (shift - shift / 2)) << 23);
                uint16_t* q = reinterpret_cast<uint16_t*>(s_x) + ((size_t)(e >> 5) * M + m) * 32 + (e & 31);
                const float f = __uint_as_float((uint32_t)*q << 16) * in1 * in2;
                *q = __half_as_ushort(__float2half_rn(f));
            }
    }
    named_bar_sync(1, kGemvConsumers);

    const int g = lane >> 2, c = lane & 3;
    const int colw = warp * 32;  // first column of this warp inside the tile
    float acc_g[MT][2][4], acc_t[MT][2][4];
#pragma unroll
    for (int a = 0; a < MT; ++a)
#pragma unroll
        for (int b2 = 0; b2 < 2; ++b2)
#pragma unroll
            for (int f = 0; f < 4; ++f) { acc_g[a][b2][f] = 0.f; acc_t[a][b2][f] = 0.f; }
    float sc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};

    int t = (int)(u0 / nb), j = j_first;
    int base = 0;  // ring row of the current unit's first word
    bool aborted = false;

    auto out_scale = [&](float v, int tok) -> float {
        if (!p.x_bf16 || s_emax[tok] == 0) return v;
        const int shift = s_emax[tok] - 141;
        return v * __int_as_float((127 + shift / 2) << 23) *
               __int_as_float((127 + (shift - shift / 2)) << 23);
    };

    auto flush = [&](int tt) {
        const int64_t ut0 = (int64_t)tt * nb;
        const int first = cta_of(ut0, G, C, W, nb, s_offs);
        const int last = cta_of(ut0 + nb - 1, G, C, W, nb, s_offs);
        const int ncol = p.N - tt * kGemvTileCols;
        if (first == last) {
#pragma unroll
            for (int ts = 0; ts < MT; ++ts)
#pragma unroll
                for (int cg = 0; cg < 2; ++cg)
#pragma unroll
                    for (int f = 0; f < 4; ++f) {
                        const int tok = ts * 8 + 2 * c + (f & 1);
                        const int cl = colw + cg * 16 + g + ((f & 2) ? 8 : 0);
                        if (tok < M && cl < ncol && !aborted)
                            p.y[(size_t)tok * p.N + (size_t)tt * kGemvTileCols + cl] =
                                __float2half_rn(out_scale(acc_t[ts][cg][f], tok));
                    }
            return;
        }
        const int which = (u0 < ut0) ? 1 : 0;
        float* my = p.slots + ((size_t)blockIdx.x * 2 + which) * (MP * kGemvTileCols);
#pragma unroll
        for (int ts = 0; ts < MT; ++ts)
#pragma unroll
            for (int cg = 0; cg < 2; ++cg)
#pragma unroll
                for (int f = 0; f < 4; ++f) {
                    const int tok = ts * 8 + 2 * c + (f & 1);
                    const int cl = colw + cg * 16 + g + ((f & 2) ? 8 : 0);
                    if (tok < M) my[tok * kGemvTileCols + cl] = out_scale(acc_t[ts][cg][f], tok);
                }
        __threadfence();
        named_bar_sync(1, kGemvConsumers);
        // A CTA between first and last whose range is empty (one unit can cost
        // more than a CTA's share) contributes nothing and is skipped.
        auto contributes = [&](int cc) {
            return unit_start(cc, G, C, W, nb, p.tiles, s_offs) <
                   unit_start(cc + 1, G, C, W, nb, p.tiles, s_offs);
        };
        if (ctid == 0) {
            int is_last = 0;
            if (!s_misc[2]) {
                int n = 0;
                for (int cc = first; cc <= last; ++cc) n += contributes(cc) ? 1 : 0;
                const int old = atomicAdd(&p.tickets[tt], 1);
                is_last = (old == n - 1);
            }
            s_misc[1] = is_last;
        }
        named_bar_sync(1, kGemvConsumers);
        if (s_misc[1]) {
            __threadfence();
            const bool first_before = (tt > 0) && cta_of(ut0 - 1, G, C, W, nb, s_offs) == first;
            for (int e = ctid; e < M * kGemvTileCols; e += kGemvConsumers) {
                const int tok = e / kGemvTileCols, cl = e - tok * kGemvTileCols;
                if (cl >= ncol) continue;
                float s = 0.f;
                for (int cc = first; cc <= last; ++cc) {
                    if (cc != first && cc != last && !contributes(cc)) continue;
                    const int wc = (cc == first && first_before) ? 1 : 0;
                    s += __ldcg(p.slots + ((size_t)cc * 2 + wc) * (MP * kGemvTileCols) +
                                tok * kGemvTileCols + cl);
                }
                p.y[(size_t)tok * p.N + (size_t)tt * kGemvTileCols + cl] = __float2half_rn(s);
            }
            if (ctid == 0) p.tickets[tt] = 0;
        }
        named_bar_sync(1, kGemvConsumers);
    };

    for (int64_t k = 0; k < nunits; ++k) {
        const int b = s_offs[j + 1] - s_offs[j];
        const bool hs = ((j & 3) == 0) || (k == 0);
        if (k > 0 && j == 0) {  // crossed into the next tile
            flush(t - 1);
#pragma unroll
            for (int a = 0; a < MT; ++a)
#pragma unroll
                for (int b2 = 0; b2 < 2; ++b2)
#pragma unroll
                    for (int f = 0; f < 4; ++f) acc_t[a][b2][f] = 0.f;
        }
        const int slot = (int)(k % kGemvSlots);
        if (!aborted) {
            if (s_misc[2] || !mbar_wait(&s_full[slot], (uint32_t)((k / kGemvSlots) & 1))) {
                aborted = true;
                s_misc[2] = 1;
            }
        }
        if (!aborted) {
            if (hs) {
                int sr = base + b;
                if (sr >= R) sr -= R;
                const __half* srow = reinterpret_cast<const __half*>(s_ring + (size_t)sr * kGemvRowBytes);
#pragma unroll
                for (int cg = 0; cg < 2; ++cg) {
                    sc[cg][0] = __half2float(srow[colw + cg * 16 + g]);
                    sc[cg][1] = __half2float(srow[colw + cg * 16 + g + 8]);
                }
            }
            int bs = j - j_first;
            if (bs < 0) bs += nb;
            uint4 xf[MT];
#pragma unroll
            for (int ts = 0; ts < MT; ++ts) {
                const int tok = ts * 8 + g;
                if (tok < M)
                    xf[ts] = *reinterpret_cast<const uint4*>(s_x + ((size_t)bs * M + tok) * 32 + c * 8);
                else
                    xf[ts] = make_uint4(0, 0, 0, 0);
            }
            switch (b) {
                case 2: unit_mma<2, MT>(s_ring, R, base, colw, g, c, xf, acc_g); break;
                case 3: unit_mma<3, MT>(s_ring, R, base, colw, g, c, xf, acc_g); break;
                case 4: unit_mma<4, MT>(s_ring, R, base, colw, g, c, xf, acc_g); break;
                case 5: unit_mma<5, MT>(s_ring, R, base, colw, g, c, xf, acc_g); break;
                case 6: unit_mma<6, MT>(s_ring, R, base, colw, g, c, xf, acc_g); break;
                default: unit_mma<8, MT>(s_ring, R, base, colw, g, c, xf, acc_g); break;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_empty[slot]);
        }
        base += b + (hs ? 1 : 0);
        if (base >= R) base -= R;
        const bool group_end = ((j & 3) == 3) || (j == nb - 1) || (k == nunits - 1);
        if (group_end) {
#pragma unroll
            for (int ts = 0; ts < MT; ++ts)
#pragma unroll
                for (int cg = 0; cg < 2; ++cg) {
                    acc_t[ts][cg][0] += sc[cg][0] * acc_g[ts][cg][0];
                    acc_t[ts][cg][1] += sc[cg][0] * acc_g[ts][cg][1];
                    acc_t[ts][cg][2] += sc[cg][1] * acc_g[ts][cg][2];
                    acc_t[ts][cg][3] += sc[cg][1] * acc_g[ts][cg][3];
#pragma unroll
                    for (int f = 0; f < 4; ++f) acc_g[ts][cg][f] = 0.f;
                }
        }
        if (++j == nb) { j = 0; ++t; }
    }
    flush(t - (j == 0 ? 1 : 0));
}

}  // namespace qg
