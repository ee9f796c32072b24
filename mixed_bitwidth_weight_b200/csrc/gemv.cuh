// Split-K GEMV for decode (M <= 16): y = x[:, perm] . dequant(Wq).
//
// The pages describe decode as bound by memory bandwidth: tokens are generated
// "as fast as memory bandwidth allows" by a kernel "near the memory-bandwidth
// limit" (navi2ai ExLlamaV3 page, "项目概述" and "核心能力").  This kernel
// streams the packed words at HBM speed on B200.  Two kernels per call:
//
// 1. xprep_kernel gathers the activations once through perm, in the order the
//    decoder emits codes (see code_of_pos), pre-scaled by 2^-P, and computes
//    a per-(block, token) correction (below).  Layout [nb][M][32] fp16 and
//    [nb][MP] fp32, so any run of blocks is one contiguous copy.
// 2. gemv_kernel, launched as a programmatic dependent of xprep_kernel: it
//    starts streaming weights at once and waits for xprep only before it
//    copies its activation span.
//
// Decode without a conversion step.  A code q at mantissa bits [P, P+b) of a
// 16-bit half ORed with 0x6400 is the fp16 number h = 1024 + q * 2^P (one
// lop3 per two codes).  With x' = x * 2^-P staged as the MMA's other operand,
// sum x' h = sum x (q - z) + sum x' (1024 + z 2^P); the second sum is the
// correction, known before the weights arrive, subtracted once per group.
// Both operands are exact fp16 values; the MMA accumulates in fp32.
//
// Work split.  W is cut into 256-column tiles; a unit is (tile, 128-row group)
// and costs the group's packed word rows.  Units are ordered tile-major and cut
// into gridDim.x contiguous ranges of equal cost (two CTAs per SM), so every SM
// streams the same number of bytes whatever the width mix.  A tile covered by
// several CTAs is finished by the last of them to arrive (an atomic ticket, no
// waiting): partial sums go to workspace slots and that CTA adds them in CTA
// order, so results are deterministic.
//
// Inside a CTA.  Warp 8 is the producer: one lane copies each unit's scale row
// and word rows with cp.async.bulk into a ring of shared-memory rows (each
// unit's rows contiguous) and signals a per-unit mbarrier.  Warps 0-7 consume,
// 32 columns each: per block a lane decodes 8 codes of each of its 4 columns
// into fp16x2 A fragments of mma.sync m16n8k16 (A = W^T tile: 16 columns x 16
// k), with the staged activations as B (16 k x 8 tokens).  The MMA cost per
// weight does not depend on M <= 16, so decode stays bound by the word stream.
#pragma once

#include "pack_dequant.cuh"

namespace qg {

constexpr int kGemvTileCols = 256;
constexpr int kGemvConsumerWarps = 8;
constexpr int kGemvConsumers = kGemvConsumerWarps * 32;
constexpr int kGemvThreads = kGemvConsumers + 32;
constexpr int kGemvRowWords = kGemvTileCols + 8;  // +8 words: rotates banks by 8 per row
constexpr int kGemvRowBytes = kGemvRowWords * 4;
constexpr int kGemvSlots = 32;                    // units in flight (mbarrier pairs)
constexpr int kGemvMaxRing = 192;                 // ring rows (cap)
constexpr int kGemvMinRing = 40;                  // one group: <= 32 word rows + 1 scale row
constexpr int kGemvGroupBlocks = kGroupRows / kBlockRows;  // 4

struct GemvParams {
    const __half* xdec;    // [nb][M][32] activations in decoder order, scaled by 2^-P
    const float* xcorr;    // [nb][MP] correction per (block, token)
    const int* xshift;     // [16] per-row power-of-two scale of bf16 input (0 for fp16)
    const uint32_t* qw;
    int64_t qw_rows;
    const __half* scales;
    const uint8_t* bits;
    const int32_t* offs;
    __half* y;
    int* tickets;          // [tiles]
    float* slots;          // [gridDim.x][2][MP][256]
    int M, K, N, nb, ng, tiles;
    int ring_rows;         // rows in the shared-memory ring
    int span_cap;          // blocks the activation stage can hold
};

struct XprepParams {
    const void* x;
    const int32_t* perm;
    const uint8_t* bits;
    const int32_t* offs;
    __half* xdec;
    float* xcorr;
    int* xshift;
    int M, K, nb, mp, x_bf16;
};

constexpr uint32_t kMagic = 0x64006400u;  // fp16x2 {1024, 1024}

// Code index (0..31 within a block) held at stage position pos = c*8 + p*2 + h:
// lane quad c, pair p of the lane's four fp16x2 registers, half h.  This is the
// order in which decode<B> emits codes.
QG_DEV int code_of_pos(int b, int pos) {
    const int c = pos >> 3, p = (pos >> 1) & 3, h = pos & 1;
    if (b == 2) return 16 * (c >> 1) + 4 * (c & 1) + p + 8 * h;
    if (b == 8) return (p < 2) ? (4 * c + p + 2 * h) : (16 + 4 * c + (p - 2) + 2 * h);
    return 8 * c + p + 4 * h;  // b = 3, 4, 5, 6
}

// Mantissa bit at which decode<B> leaves the code of stage position pos.
QG_DEV int shift_of_pos(int b, int pos) {
    const int p = (pos >> 1) & 3;
    switch (b) {
        case 2: return 2 * p;
        case 3: return (p == 1) ? 3 : (p == 2) ? 6 : 0;
        case 4: return (p & 1) ? 4 : 0;
        case 5: return (p & 1) ? 5 : 0;
        default: return 0;  // 6 and 8
    }
}

// Word rows decode4<B> reads for lane quad c (relative to the block's first
// word row): lo_row and hi_row (hi_row == lo_row when one row suffices).
template <int B>
QG_DEV int lo_row(int c) {
    if constexpr (B == 2) return c >> 1;
    else if constexpr (B == 3) return c <= 1 ? 0 : c - 1;
    else if constexpr (B == 6) return c < 2 ? c : c + 1;
    else return c;  // 4, 5, 8
}
template <int B>
QG_DEV int hi_row(int c) {
    if constexpr (B == 3) return c <= 1 ? 1 : 2;
    else if constexpr (B == 5) return c + 1;
    else if constexpr (B == 6) return (c < 2 ? c : c + 1) + 1;
    else if constexpr (B == 8) return c + 4;
    else return lo_row<B>(c);  // 2, 4
}

// The 8 codes lane quad c owns in each of its 4 adjacent columns, as fp16x2
// values h = 1024 + q * 2^P.  wlo / whi point at the lane's words (rows lo_row
// and hi_row of the block) of its first column; the 4 columns are one 16-byte
// load.  P[q][p] = pair p of column q.
template <int B>
QG_DEV void decode4(const uint8_t* wlo, const uint8_t* whi, int c, uint32_t (&P)[4][4]) {
    auto col = [](const uint4& v, int q) { return q == 0 ? v.x : q == 1 ? v.y : q == 2 ? v.z : v.w; };
    const uint4 rl = *reinterpret_cast<const uint4*>(wlo);
    if constexpr (B == 2) {
        const int sh = (c & 1) * 8;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t v = col(rl, q) >> sh;
            P[q][0] = lop3_mask_magic<0x00030003u>(v);
            P[q][1] = lop3_mask_magic<0x000C000Cu>(v);
            P[q][2] = lop3_mask_magic<0x00300030u>(v);
            P[q][3] = lop3_mask_magic<0x00C000C0u>(v);
        }
    } else if constexpr (B == 3) {
        const uint4 rh = *reinterpret_cast<const uint4*>(whi);
        const int s0 = (c == 0) ? 0 : 32 - 8 * c;  // 0, 24, 16, 8
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t X = __funnelshift_r(col(rl, q), col(rh, q), s0);  // codes i at 3i
            const uint32_t u = (X & 0xFFFFu) | ((X << 4) & 0xFFFF0000u);
            P[q][0] = lop3_mask_magic<0x00070007u>(u);
            P[q][1] = lop3_mask_magic<0x00380038u>(u);
            P[q][2] = lop3_mask_magic<0x01C001C0u>(u);
            P[q][3] = lop3_mask_magic<0x00070007u>(u >> 9);
        }
    } else if constexpr (B == 4) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t v = col(rl, q), v2 = v >> 8;
            P[q][0] = lop3_mask_magic<0x000F000Fu>(v);
            P[q][1] = lop3_mask_magic<0x00F000F0u>(v);
            P[q][2] = lop3_mask_magic<0x000F000Fu>(v2);
            P[q][3] = lop3_mask_magic<0x00F000F0u>(v2);
        }
    } else if constexpr (B == 5) {
        const uint4 rh = *reinterpret_cast<const uint4*>(whi);
        const int s0 = (8 * c) & 31;  // 40c mod 32
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint64_t X = ((((uint64_t)col(rh, q)) << 32) | col(rl, q)) >> s0;  // codes i at 5i
            const uint32_t u1 = prmt_i<0x5410>((uint32_t)X, (uint32_t)(X >> 20));
            const uint32_t u2 = prmt_i<0x5410>((uint32_t)(X >> 10), (uint32_t)(X >> 30));
            P[q][0] = lop3_mask_magic<0x001F001Fu>(u1);
            P[q][1] = lop3_mask_magic<0x03E003E0u>(u1);
            P[q][2] = lop3_mask_magic<0x001F001Fu>(u2);
            P[q][3] = lop3_mask_magic<0x03E003E0u>(u2);
        }
    } else if constexpr (B == 6) {
        const uint4 rh = *reinterpret_cast<const uint4*>(whi);
        const int s0 = (c & 1) * 16;  // 0, 16, 0, 16
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint64_t X = ((((uint64_t)col(rh, q)) << 32) | col(rl, q)) >> s0;  // codes i at 6i
#pragma unroll
            for (int i = 0; i < 4; ++i)
                P[q][i] = lop3_mask_magic<0x003F003Fu>(
                    prmt_i<0x5410>((uint32_t)(X >> (6 * i)), (uint32_t)(X >> (6 * i + 24))));
        }
    } else {  // B == 8
        const uint4 rh = *reinterpret_cast<const uint4*>(whi);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            P[q][0] = prmt_i<0x4240>(col(rl, q), 0x64646464u);
            P[q][1] = prmt_i<0x4341>(col(rl, q), 0x64646464u);
            P[q][2] = prmt_i<0x4240>(col(rh, q), 0x64646464u);
            P[q][3] = prmt_i<0x4341>(col(rh, q), 0x64646464u);
        }
    }
}

// One block: decode the lane's 4 columns and run 2 x MT mma.sync per column
// pair.  The lane's columns colq..colq+3 are the A-fragment rows (g, g+8) of
// column group 0 and (g, g+8) of column group 1.  FIRST starts the accumulators.
template <int B, int MT, bool FIRST>
QG_DEV void block_mma(const uint8_t* wlo, const uint8_t* whi, int c, const uint4 (&xf)[MT],
                      float (&acc)[MT][2][4]) {
    uint32_t P[4][4];
    decode4<B>(wlo, whi, c, P);
#pragma unroll
    for (int cg = 0; cg < 2; ++cg)
#pragma unroll
        for (int ts = 0; ts < MT; ++ts) {
            if (FIRST)
                mma_f16_16816_first(acc[ts][cg], P[2 * cg][0], P[2 * cg + 1][0], P[2 * cg][1],
                                    P[2 * cg + 1][1], xf[ts].x, xf[ts].y);
            else
                mma_f16_16816(acc[ts][cg], P[2 * cg][0], P[2 * cg + 1][0], P[2 * cg][1], P[2 * cg + 1][1],
                              xf[ts].x, xf[ts].y);
            mma_f16_16816(acc[ts][cg], P[2 * cg][2], P[2 * cg + 1][2], P[2 * cg][3], P[2 * cg + 1][3],
                          xf[ts].z, xf[ts].w);
        }
}

// Activation fragments of one block record for the lane's tokens (g, g + 8).
template <int MT>
QG_DEV void load_xf(const uint8_t* xrec, const bool (&xv)[2], uint4 (&xf)[MT]) {
#pragma unroll
    for (int ts = 0; ts < MT; ++ts)
        xf[ts] = xv[ts] ? *reinterpret_cast<const uint4*>(xrec + ts * 8 * 64) : make_uint4(0, 0, 0, 0);
}

// A full group whose 4 blocks share width B: every word offset is a constant
// added to the lane's two row pointers.  w0 = first word row of the group at
// the lane's first column; xrec = the lane's record of the group's block 0.
// Even and odd blocks accumulate separately (shorter MMA dependency chains).
template <int B, int MT>
QG_DEV void group_mma(const uint8_t* w0, const uint8_t* xrec, int xstride, int c, const bool (&xv)[2],
                      float (&acc)[MT][2][4]) {
    const uint8_t* wlo = w0 + lo_row<B>(c) * kGemvRowBytes;
    const uint8_t* whi = w0 + hi_row<B>(c) * kGemvRowBytes;
    float acc2[MT][2][4];
    uint4 xa[MT], xb[MT];
    load_xf<MT>(xrec, xv, xa);
    load_xf<MT>(xrec + xstride, xv, xb);
    block_mma<B, MT, true>(wlo, whi, c, xa, acc);
    block_mma<B, MT, true>(wlo + B * kGemvRowBytes, whi + B * kGemvRowBytes, c, xb, acc2);
    load_xf<MT>(xrec + 2 * xstride, xv, xa);
    load_xf<MT>(xrec + 3 * xstride, xv, xb);
    block_mma<B, MT, false>(wlo + 2 * B * kGemvRowBytes, whi + 2 * B * kGemvRowBytes, c, xa, acc);
    block_mma<B, MT, false>(wlo + 3 * B * kGemvRowBytes, whi + 3 * B * kGemvRowBytes, c, xb, acc2);
#pragma unroll
    for (int ts = 0; ts < MT; ++ts)
#pragma unroll
        for (int cg = 0; cg < 2; ++cg)
#pragma unroll
            for (int f = 0; f < 4; ++f) acc[ts][cg][f] += acc2[ts][cg][f];
}

// One block of any width (groups with mixed widths or fewer than 4 blocks).
template <int B, int MT>
QG_DEV void any_block_mma(const uint8_t* wb, const uint8_t* xrec, int c, const bool (&xv)[2],
                          float (&acc)[MT][2][4]) {
    uint4 xf[MT];
    load_xf<MT>(xrec, xv, xf);
    block_mma<B, MT, false>(wb + lo_row<B>(c) * kGemvRowBytes, wb + hi_row<B>(c) * kGemvRowBytes, c, xf, acc);
}

// Units are numbered t*ng + g.  A unit's cost is its word rows plus its scale
// row, so the cost prefix of (t, g) is t*(W + ng) + offs[4g] + g, with W the
// word rows of one tile.  CTA i owns the units whose prefix lies in
// [ceil(i*C/G), ceil((i+1)*C/G)), C = tiles * (W + ng).
QG_DEV int64_t unit_start(int64_t i, int64_t G, int64_t C, int64_t W, int nb, int ng, int tiles,
                          const int32_t* s_offs) {
    if (i >= G) return (int64_t)tiles * ng;
    const int64_t Wt = W + ng;
    int64_t t, rem;
    if (C * G < (1ll << 32)) {  // the usual case: 32-bit division
        const uint32_t pos = ((uint32_t)i * (uint32_t)C + (uint32_t)G - 1u) / (uint32_t)G;
        t = pos / (uint32_t)Wt;
        rem = pos - (uint32_t)t * (uint32_t)Wt;
    } else {
        const int64_t pos = (i * C + G - 1) / G;
        t = pos / Wt;
        rem = pos - t * Wt;
    }
    int lo = 0, hi = ng;  // first g in [0, ng] with offs[min(4g, nb)] + g >= rem
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (s_offs[min(mid * kGemvGroupBlocks, nb)] + mid >= rem) hi = mid; else lo = mid + 1;
    }
    return t * ng + lo;  // lo == ng rolls over to the next tile's group 0
}

// CTA that owns unit u.
QG_DEV int cta_of(int64_t u, int64_t G, int64_t C, int64_t W, int ng, const int32_t* s_offs) {
    const int64_t t = u / ng;
    const int g = (int)(u - t * ng);
    const int64_t pos = t * (W + ng) + s_offs[g * kGemvGroupBlocks] + g;
    if (C * G < (1ll << 32)) return (int)(((uint32_t)pos * (uint32_t)G) / (uint32_t)C);
    return (int)((pos * G) / C);
}

// Ring rows of a unit: its scale row and word rows, contiguous; a unit that
// would cross the end of the ring starts at row 0 instead.  `pos` is the next
// free row, `total` a monotone count of rows used (skipped tails included);
// producer and consumers replay the same sequence.
QG_DEV int ring_alloc(int& pos, int64_t& total, int need, int R) {
    if (pos + need > R) {
        total += R - pos;
        pos = 0;
    }
    const int r = pos;
    pos += need;
    total += need;
    return r;
}

// ------------------------------------------------------------------ xprep
// One warp per (block, token): lane = stage position.  Writes the decoder-
// order activation (scaled by 2^-P); the correction sum x' * (1024 + z * 2^P)
// is reduced per 128-row group (8 warps = 2 groups per CTA).  bf16 input is
// first scaled per row by 2^-shift so that the row's largest magnitude lands in
// [2^14, 2^15).
__global__ void __launch_bounds__(256) xprep_kernel(const XprepParams p) {
    asm volatile("griddepcontrol.launch_dependents;");
    __shared__ int s_shift[16];
    __shared__ float s_bc[8][16];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x < 16) s_shift[threadIdx.x] = 0;
    __syncthreads();
    if (p.x_bf16) {
        // full-row maximum exponent of every token row (rows are short)
        for (int m = 0; m < p.M; ++m) {
            int e = 0;
            const uint16_t* row = reinterpret_cast<const uint16_t*>(p.x) + (size_t)m * p.K;
            for (int k = threadIdx.x; k < p.K; k += blockDim.x) e = max(e, (int)((row[k] >> 7) & 0xFF));
#pragma unroll
            for (int o = 16; o; o >>= 1) e = max(e, __shfl_xor_sync(0xffffffffu, e, o));
            if (lane == 0) atomicMax(&s_shift[m], e);
        }
        __syncthreads();
        if (threadIdx.x < p.M) {
            const int e = s_shift[threadIdx.x];
            s_shift[threadIdx.x] = (e == 0) ? 0 : e - 141;
        }
        __syncthreads();
    }
    if (blockIdx.x == 0 && threadIdx.x < 16) p.xshift[threadIdx.x] = s_shift[threadIdx.x];
    const int j = blockIdx.x * 8 + warp;
    const int b = (j < p.nb) ? (int)p.bits[j] : 2;
    const bool live = (j < p.nb) && width_ok(b);
    if (j < p.nb && !width_ok(b) && lane == 0) set_dev_error(QGEMM_DEV_BAD_SCHEDULE);
    int src = 0;
    int P = 0;
    if (live) {
        P = shift_of_pos(b, lane);
        src = p.perm[j * kBlockRows + code_of_pos(b, lane)];
        if (src < 0 || src >= p.K) {
            set_dev_error(QGEMM_DEV_BAD_PERM);
            src = 0;
        }
    }
    const float offset = (float)(1024 + (1 << (b - 1)) * (1 << P));
    const float inv2p = __int_as_float((127 - P) << 23);
    for (int m = 0; m < p.M; ++m) {
        float corr = 0.f;
        if (live) {
            const uint16_t raw = reinterpret_cast<const uint16_t*>(p.x)[(size_t)m * p.K + src];
            float v;
            if (p.x_bf16) {
                const int sh = s_shift[m];
                v = __uint_as_float((uint32_t)raw << 16) * __int_as_float((127 - sh / 2) << 23) *
                    __int_as_float((127 - (sh - sh / 2)) << 23);
            } else {
                v = __half2float(__ushort_as_half(raw));
            }
            const __half xs = __float2half_rn(v * inv2p);  // exact unless below fp16 normals
            p.xdec[((size_t)j * p.M + m) * kBlockRows + lane] = xs;
            corr = __half2float(xs) * offset;
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) corr += __shfl_xor_sync(0xffffffffu, corr, o);
        if (lane == 0) s_bc[warp][m] = corr;
    }
    __syncthreads();
    // group gl of this CTA = blocks 4gl..4gl+3 = warps 4gl..4gl+3
    if (threadIdx.x < 2 * p.M) {
        const int gl = threadIdx.x / p.M, m = threadIdx.x - gl * p.M;
        const int gg = blockIdx.x * 2 + gl;
        if (gg * kGemvGroupBlocks < p.nb)
            p.xcorr[(size_t)gg * p.mp + m] = s_bc[4 * gl][m] + s_bc[4 * gl + 1][m] +
                                              s_bc[4 * gl + 2][m] + s_bc[4 * gl + 3][m];
    }
}

// -------------------------------------------------------------------- GEMV
template <int MT>
__global__ void __launch_bounds__(kGemvThreads, (MT == 1) ? 2 : 1) gemv_kernel(const GemvParams p) {
    constexpr int MP = MT * 8;
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nb = p.nb, ng = p.ng, M = p.M;

    int32_t* s_offs = reinterpret_cast<int32_t*>(smem);
    size_t o = ((size_t)(nb + 1) * 4 + 15) & ~(size_t)15;
    uint64_t* s_full = reinterpret_cast<uint64_t*>(smem + o);
    o += kGemvSlots * 8;
    uint64_t* s_empty = reinterpret_cast<uint64_t*>(smem + o);
    o += kGemvSlots * 8;
    uint64_t* s_xfull = reinterpret_cast<uint64_t*>(smem + o);
    o += 16;
    int* s_misc = reinterpret_cast<int*>(smem + o);  // bad schedule, last flag, abort, shifts
    int* s_shift = s_misc + 16;
    o += 128;
    __half* s_x = reinterpret_cast<__half*>(smem + o);
    o += (size_t)p.span_cap * M * 64;
    float* s_corr = reinterpret_cast<float*>(smem + o);  // per group
    o += (size_t)((p.span_cap + kGemvGroupBlocks - 1) / kGemvGroupBlocks + 1) * MP * 4;
    o = (o + 15) & ~(size_t)15;
    uint8_t* s_ring = smem + o;
    const int R = p.ring_rows;

    // ---- schedule into shared memory (one round trip), validated before any
    // weight access: widths allowed and offsets equal to their prefix sums
    if (tid < 32) s_misc[tid] = 0;
    int32_t my_off[4], my_next[4];
    uint8_t my_bits[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int j = tid + q * kGemvThreads;
        my_off[q] = (j <= nb) ? p.offs[j] : 0;
        my_next[q] = (j < nb) ? p.offs[j + 1] : 0;
        my_bits[q] = (j < nb) ? p.bits[j] : (uint8_t)2;
    }
    for (int j = tid + 4 * kGemvThreads; j <= nb; j += kGemvThreads) s_offs[j] = p.offs[j];
    bool bad = false;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int j = tid + q * kGemvThreads;
        if (j <= nb) s_offs[j] = my_off[q];
        if (j < nb && (!width_ok(my_bits[q]) || my_next[q] - my_off[q] != my_bits[q])) bad = true;
    }
    for (int j = tid + 4 * kGemvThreads; j < nb; j += kGemvThreads) {
        const int b = p.bits[j];
        if (!width_ok(b) || p.offs[j + 1] - p.offs[j] != b) bad = true;
    }
    if (tid == 0 && (my_off[0] != 0 || (int64_t)p.offs[nb] != p.qw_rows)) bad = true;
    __syncthreads();
    if (bad) atomicOr(&s_misc[0], 1);
    if (tid == 0) {
        for (int i = 0; i < kGemvSlots; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&s_empty[i], kGemvConsumerWarps);
        }
        mbar_init(s_xfull, 1);
        fence_mbar_init();
    }
    __syncthreads();
    // Every early exit waits for the xprep grid first, so this grid never
    // completes before the one it depends on.
    if (s_misc[0]) {
        if (tid == 0) {
            set_dev_error(QGEMM_DEV_BAD_SCHEDULE);
            asm volatile("griddepcontrol.wait;" ::: "memory");
        }
        return;
    }

    const int64_t W = s_offs[nb];
    const int64_t C = (int64_t)p.tiles * (W + ng);
    const int64_t G = gridDim.x;
    const int64_t u0 = unit_start(blockIdx.x, G, C, W, nb, ng, p.tiles, s_offs);
    const int64_t u1 = unit_start(blockIdx.x + 1, G, C, W, nb, ng, p.tiles, s_offs);
    const int nunits = (int)(u1 - u0);
    if (nunits <= 0) {
        if (tid == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
        return;
    }
    const int t0 = (int)(u0 / ng), gf = (int)(u0 - (int64_t)t0 * ng);  // first unit (tile, group)
    const int jf = gf * kGemvGroupBlocks;  // block window [jf, jf + span) mod nb
    const int gspan = min(ng, nunits);     // group window [gf, gf + gspan) mod ng
    int span;
    {
        int blocks = 0, g = gf;
        for (int k = 0; k < gspan; ++k) {
            blocks += min(kGemvGroupBlocks, nb - g * kGemvGroupBlocks);
            if (++g == ng) g = 0;
        }
        span = min(blocks, nb);
    }

    // =================================================== producer warp
    if (warp == kGemvConsumerWarps) {
        if (lane != 0) return;
        const uint64_t policy = policy_evict_first();
        int pos = 0, pos_rel = 0;
        int64_t total = 0, total_rel = 0;
        int k_rel = 0, g_rel = gf;
        bool ok = true;
        bool x_issued = false;
        int k = 0;
        auto issue_x = [&]() {
            // activations and corrections of the CTA's windows (1 or 2 runs
            // each); they are written by the preceding xprep grid
            asm volatile("griddepcontrol.wait;" ::: "memory");
            const int brun = min(span, nb - jf), grun = min(gspan, ng - gf);
            const uint32_t xbytes = (uint32_t)span * M * 64 + (uint32_t)gspan * MP * 4;
            mbar_arrive_expect_tx(s_xfull, xbytes);
            bulk_g2s(s_x, p.xdec + (size_t)jf * M * kBlockRows, (uint32_t)brun * M * 64, s_xfull);
            if (brun < span)
                bulk_g2s(s_x + (size_t)brun * M * kBlockRows, p.xdec, (uint32_t)(span - brun) * M * 64,
                         s_xfull);
            bulk_g2s(s_corr, p.xcorr + (size_t)gf * MP, (uint32_t)grun * MP * 4, s_xfull);
            if (grun < gspan)
                bulk_g2s(s_corr + (size_t)grun * MP, p.xcorr, (uint32_t)(gspan - grun) * MP * 4, s_xfull);
            x_issued = true;
        };
        int t = t0, g = gf;
        for (; k < nunits && ok; ++k) {
            const int j0 = g * kGemvGroupBlocks, j1 = min(j0 + kGemvGroupBlocks, nb);
            const int wrows = s_offs[j1] - s_offs[j0];
            const int need = wrows + 1;
            // wait until the ring has room and a barrier slot is free
            int ppos = pos;
            int64_t ptotal = total;
            ring_alloc(ppos, ptotal, need, R);
            while (k - k_rel >= kGemvSlots || ptotal - total_rel > R) {
                if (!x_issued) issue_x();  // nothing else to do while waiting
                if (!mbar_wait(&s_empty[k_rel & (kGemvSlots - 1)], (uint32_t)((k_rel / kGemvSlots) & 1))) {
                    ok = false;
                    break;
                }
                const int jr0 = g_rel * kGemvGroupBlocks, jr1 = min(jr0 + kGemvGroupBlocks, nb);
                ring_alloc(pos_rel, total_rel, s_offs[jr1] - s_offs[jr0] + 1, R);
                ++k_rel;
                if (++g_rel == ng) g_rel = 0;
            }
            if (!ok) break;
            const int row = ring_alloc(pos, total, need, R);
            const int slot = k & (kGemvSlots - 1);
            const int cols = min(kGemvTileCols, p.N - t * kGemvTileCols);
            mbar_arrive_expect_tx(&s_full[slot], (uint32_t)(cols * 2 + wrows * cols * 4));
            uint8_t* dst = s_ring + (size_t)row * kGemvRowBytes;
            bulk_g2s(dst, p.scales + (size_t)g * p.N + (size_t)t * kGemvTileCols, (uint32_t)cols * 2,
                     &s_full[slot]);
            const uint32_t* src = p.qw + (size_t)s_offs[j0] * p.N + (size_t)t * kGemvTileCols;
            for (int r = 0; r < wrows; ++r)
                bulk_g2s_hint(dst + (size_t)(r + 1) * kGemvRowBytes, src + (size_t)r * p.N,
                              (uint32_t)cols * 4, &s_full[slot], policy);
            if (++g == ng) { g = 0; ++t; }
        }
        if (ok && !x_issued) issue_x();
        if (!ok) {
            if (!x_issued) asm volatile("griddepcontrol.wait;" ::: "memory");
            s_misc[2] = 1;
            // let copies already in flight land before the CTA can exit
            for (int kk = k_rel; kk < k; ++kk)
                mbar_wait(&s_full[kk & (kGemvSlots - 1)], (uint32_t)((kk / kGemvSlots) & 1));
            if (x_issued) mbar_wait(s_xfull, 0);
        }
        return;
    }

    // =================================================== consumer warps
    const int ctid = tid;  // 0..255
    const int g8 = lane >> 2, c = lane & 3;
    const int colw = warp * 32;       // first column of this warp inside the tile
    const int colq = colw + 4 * g8;   // the lane's 4 columns: A rows (g, g+8) of groups 0, 1
    float acc_g[MT][2][4], acc_t[MT][2][4];
#pragma unroll
    for (int a = 0; a < MT; ++a)
#pragma unroll
        for (int b2 = 0; b2 < 2; ++b2)
#pragma unroll
            for (int f = 0; f < 4; ++f) { acc_g[a][b2][f] = 0.f; acc_t[a][b2][f] = 0.f; }
    bool aborted = false;
    if (!mbar_wait(s_xfull, 0)) {
        aborted = true;
        s_misc[2] = 1;
    }
    if (ctid < 16) s_shift[ctid] = p.xshift[ctid];
    named_bar_sync(1, kGemvConsumers);

    auto out_scale = [&](float v, int tok) -> float {
        const int sh = s_shift[tok];
        if (sh == 0) return v;
        return v * __int_as_float((127 + sh / 2) << 23) * __int_as_float((127 + (sh - sh / 2)) << 23);
    };

    // C fragment element f of column pair cg: token ts*8 + 2c + (f & 1),
    // column colq + 2*cg + (f >> 1).
    auto flush = [&](int tt) {
        const int64_t ut0 = (int64_t)tt * ng;
        const int first = cta_of(ut0, G, C, W, ng, s_offs);
        const int last = cta_of(ut0 + ng - 1, G, C, W, ng, s_offs);
        const int ncol = p.N - tt * kGemvTileCols;
        if (first == last) {
#pragma unroll
            for (int ts = 0; ts < MT; ++ts)
#pragma unroll
                for (int cg = 0; cg < 2; ++cg)
#pragma unroll
                    for (int f = 0; f < 4; ++f) {
                        const int tok = ts * 8 + 2 * c + (f & 1);
                        const int cl = colq + 2 * cg + (f >> 1);
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
                    const int cl = colq + 2 * cg + (f >> 1);
                    if (tok < M) my[tok * kGemvTileCols + cl] = out_scale(acc_t[ts][cg][f], tok);
                }
        __threadfence();
        named_bar_sync(1, kGemvConsumers);
        if (ctid == 0) {
            // every CTA in [first, last] owns a unit of this tile: the host sizes
            // the grid so that no CTA's range is empty
            int is_last = 0;
            if (!s_misc[2]) is_last = (atomicAdd(&p.tickets[tt], 1) == last - first);
            s_misc[1] = is_last;
        }
        named_bar_sync(1, kGemvConsumers);
        if (s_misc[1]) {
            __threadfence();
            const bool first_before = (tt > 0) && cta_of(ut0 - 1, G, C, W, ng, s_offs) == first;
            for (int e = ctid; e < M * kGemvTileCols; e += kGemvConsumers) {
                const int tok = e / kGemvTileCols, cl = e - tok * kGemvTileCols;
                if (cl >= ncol) continue;
                float s = 0.f;
                for (int cc = first; cc <= last; ++cc) {
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

    const int xstride = M * 64;                           // bytes per block record
    const uint8_t* s_x8 = reinterpret_cast<const uint8_t*>(s_x) + (g8 * 32 + c * 8) * 2;
    const bool xv[2] = {g8 < M, 8 + g8 < M};
    int pos = 0;
    int64_t total = 0;
    int t = t0, g = gf, t_prev = t0, bs0 = 0, gs = 0;  // bs0: stage block of the group's block 0
    for (int k = 0; k < nunits; ++k) {
        if (t != t_prev) {  // crossed into the next tile
            flush(t_prev);
            t_prev = t;
#pragma unroll
            for (int a = 0; a < MT; ++a)
#pragma unroll
                for (int b2 = 0; b2 < 2; ++b2)
#pragma unroll
                    for (int f = 0; f < 4; ++f) acc_t[a][b2][f] = 0.f;
        }
        const int j0 = g * kGemvGroupBlocks, j1 = min(j0 + kGemvGroupBlocks, nb);
        const int o0 = s_offs[j0];
        const int row = ring_alloc(pos, total, s_offs[j1] - o0 + 1, R);
        const int slot = k & (kGemvSlots - 1);
        bool go = !aborted;
        if (go && (s_misc[2] || !mbar_wait(&s_full[slot], (uint32_t)((k / kGemvSlots) & 1)))) {
            aborted = true;
            s_misc[2] = 1;
            go = false;
        }
        if (go) {
            const uint8_t* ub = s_ring + (size_t)row * kGemvRowBytes;
            const uint2 sv = *reinterpret_cast<const uint2*>(ub + colq * 2);
            const uint8_t* w0 = ub + kGemvRowBytes + colq * 4;
            const uint8_t* xrec = s_x8 + bs0 * xstride;
            const int b0 = s_offs[j0 + 1] - o0;
            const bool uniform = (j1 - j0 == kGemvGroupBlocks) && (s_offs[j1] - o0 == 4 * b0) &&
                                 (s_offs[j0 + 2] - o0 == 2 * b0) && (s_offs[j0 + 3] - o0 == 3 * b0);
            if (uniform) {
                switch (b0) {
                    case 2: group_mma<2, MT>(w0, xrec, xstride, c, xv, acc_g); break;
                    case 3: group_mma<3, MT>(w0, xrec, xstride, c, xv, acc_g); break;
                    case 4: group_mma<4, MT>(w0, xrec, xstride, c, xv, acc_g); break;
                    case 5: group_mma<5, MT>(w0, xrec, xstride, c, xv, acc_g); break;
                    case 6: group_mma<6, MT>(w0, xrec, xstride, c, xv, acc_g); break;
                    default: group_mma<8, MT>(w0, xrec, xstride, c, xv, acc_g); break;
                }
            } else {
#pragma unroll
                for (int a = 0; a < MT; ++a)
#pragma unroll
                    for (int b2 = 0; b2 < 2; ++b2)
#pragma unroll
                        for (int f = 0; f < 4; ++f) acc_g[a][b2][f] = 0.f;
                for (int j = j0; j < j1; ++j) {
                    const int b = s_offs[j + 1] - s_offs[j];
                    const uint8_t* wb = w0 + (s_offs[j] - o0) * kGemvRowBytes;
                    const uint8_t* xr = xrec + (j - j0) * xstride;
                    switch (b) {
                        case 2: any_block_mma<2, MT>(wb, xr, c, xv, acc_g); break;
                        case 3: any_block_mma<3, MT>(wb, xr, c, xv, acc_g); break;
                        case 4: any_block_mma<4, MT>(wb, xr, c, xv, acc_g); break;
                        case 5: any_block_mma<5, MT>(wb, xr, c, xv, acc_g); break;
                        case 6: any_block_mma<6, MT>(wb, xr, c, xv, acc_g); break;
                        default: any_block_mma<8, MT>(wb, xr, c, xv, acc_g); break;
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_empty[slot]);
            // group done: remove the offset terms, apply the (group, column) scale
            float sc[2][2];
            sc[0][0] = __low2float(*reinterpret_cast<const __half2*>(&sv.x));
            sc[0][1] = __high2float(*reinterpret_cast<const __half2*>(&sv.x));
            sc[1][0] = __low2float(*reinterpret_cast<const __half2*>(&sv.y));
            sc[1][1] = __high2float(*reinterpret_cast<const __half2*>(&sv.y));
#pragma unroll
            for (int ts = 0; ts < MT; ++ts) {
                const float2 cr = *reinterpret_cast<const float2*>(s_corr + (size_t)gs * MP + ts * 8 + 2 * c);
#pragma unroll
                for (int cg = 0; cg < 2; ++cg) {
                    acc_t[ts][cg][0] += sc[cg][0] * (acc_g[ts][cg][0] - cr.x);
                    acc_t[ts][cg][1] += sc[cg][0] * (acc_g[ts][cg][1] - cr.y);
                    acc_t[ts][cg][2] += sc[cg][1] * (acc_g[ts][cg][2] - cr.x);
                    acc_t[ts][cg][3] += sc[cg][1] * (acc_g[ts][cg][3] - cr.y);
                }
            }
        }
        // next unit
        bs0 += j1 - j0;
        if (bs0 >= nb) bs0 -= nb;
        if (++gs == ng) gs = 0;
        if (++g == ng) { g = 0; ++t; }
    }
    flush(t_prev);
}

}  // namespace qg
