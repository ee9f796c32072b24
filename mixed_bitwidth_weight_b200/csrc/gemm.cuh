// Prefill GEMM on the 5th-generation tensor cores: y = x[:, perm] . dequant(Wq)
// for M > 16 (the quantised GEMM of the exllamav2 report, "解法哲学", which
// the pages credit with near-bandwidth decode and tensor-core prefill).
//
// Two kernels:
// * xperm_kernel writes x_p = x[:, perm] (the act-order gather) into the
//   workspace as fp16, so that the activation tiles are plain 2D boxes and
//   both MMA operands are fp16 (bf16 input is scaled per row by a power of
//   two first, exactly, and y is scaled back).
// * gemm_kernel computes one 256 x 256 tile of y per CTA.  Warp roles:
//     warp 0     - activation producer: per 64-row k step the activation
//                  tile (256 rows x 64 k, 128-byte swizzle; only its 64-row
//                  slices that hold rows of x when there are fewer);
//     warp 1     - allocates TMEM (two 128 x 256 fp32 accumulators, all 512
//                  columns) and issues the MMAs from one thread:
//                  tcgen05.mma kind::f16, M = 128, N = 256, K = 16, both
//                  operands from shared memory;
//     warps 2-17 - dequantise: thread (n, k) decodes the 32 codes of column n
//                  in block k of the step (each block at its own width) two
//                  per instruction in fp16 pairs, forms w = (q - 2^(b-1)) * s
//                  with one rounding (the bit-exact dequantised weight) and
//                  writes row n of the B tile in the
//                  K-major 128-byte-swizzled layout the MMA reads; after the
//                  last step they move the accumulators TMEM -> fp16 y;
//     warp 18    - word-row producer: per k step the step's word rows (2D
//                  boxes) and its group's scale row (a warp of its own, so
//                  the two copy streams wait only on their own stages).
// Every wait is bounded; a timeout sets the device error word, the CTA skips
// the remaining work, waits for its copies and MMAs and frees TMEM.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "pack_dequant.cuh"

namespace qg {

constexpr int kGemmBM = 256;
constexpr int kGemmBN = 256;
constexpr int kGemmBK = 64;                              // two 32-row blocks per k step
constexpr int kGemmAStages = 3;
constexpr int kGemmBStages = 2;
constexpr int kGemmRStages = 3;
constexpr int kGemmABytes = kGemmBM * kGemmBK * 2;       // 32 KB
constexpr int kGemmBBytes = kGemmBN * kGemmBK * 2;       // 32 KB
constexpr int kGemmRawRows = 16;                         // word rows of two blocks, at most
constexpr int kGemmRBytes = (kGemmRawRows + 1) * 1024;   // scale row + word rows
constexpr int kGemmDecWarps = 16;                        // 2 blocks x 256 columns per k step
constexpr int kGemmRawWarp = 2 + kGemmDecWarps;          // the word-row producer (last warp)
constexpr int kGemmThreads = 64 + kGemmDecWarps * 32 + 32;
constexpr int kGemmBoxMaps = 5;                          // word boxes of 1, 2, 4, 8, 16 rows
constexpr int kGemmMaxSplit = 4;                         // k splits of one tile, at most
constexpr int kGemmFixedSmem =
    kGemmAStages * kGemmABytes + kGemmBStages * kGemmBBytes + kGemmRStages * kGemmRBytes + 1024;

struct GemmMaps {
    CUtensorMap a;                    // x_p [M][K], box {64, 256}, 128-byte swizzle
    CUtensorMap a64;                  // the same with box {64, 64}: tiles with few rows of x
    CUtensorMap w[kGemmBoxMaps];      // qw [qw_rows][N], box {256, 2^i}
};

struct GemmParams {
    const int* xshift;   // [M] row shifts of bf16 input (x_bf16 != 0)
    const __half* scales;
    const uint8_t* bits;
    const int32_t* offs;
    int64_t qw_rows;
    __half* y;
    int* tickets;      // [tiles] (split tiles only)
    float* partial;    // [split tiles][ksplit][256][256] fp32 partial sums
    int M, K, N, nb, mtiles, ntiles, x_bf16;
    int full_tiles;    // tiles done whole, one per CTA (whole waves of the grid)
    int ksplit;        // k splits of each remaining tile (the last wave)
};

struct XpermParams {
    const uint16_t* x;
    const int32_t* perm;
    const uint8_t* bits;
    uint16_t* xp;
    int* xshift;   // [M] per-row power-of-two shift (bf16 input)
    int M, K, x_bf16;
};

// Codes paired into one fp16x2 word by the dequantiser: pair i of a block
// holds codes r = 2m (i / m) + i % m (low half) and r + m (high half), so
// that one 32-bit window of the block's bit stream holds both, r at window
// bit kl and r + m at bit 16 + kh (pair_kl / pair_kh below): m = 8, 4, 2 for
// b = 2, 4, 8 (the codes 16 bits apart), m = 4 for b = 3 and 5, 2 for b = 6.
QG_DEV constexpr int pair_m(int b) { return b == 2 ? 8 : (b == 6 || b == 8) ? 2 : 4; }
QG_DEV constexpr int pair_kl(int b) { return (b == 3 || b == 6) ? 4 : 0; }
QG_DEV constexpr int pair_kh(int b) { return b == 5 ? 4 : 0; }

// Order of the k positions of one 32-row block inside the B tile (and so in
// x_p): position 2i + h holds code r + h m of pair i.
QG_DEV int gemm_code_of_k(int b, int k) {
    const int i = k >> 1, h = k & 1, m = pair_m(b);
    return 2 * m * (i / m) + i % m + m * h;
}

// x_p[m][k] = fp16(x[m][perm[k']] * 2^-shift[m]), k' = the code the B tile
// holds at position k (gemm_code_of_k).  One CTA per kXpermRows rows (and
// per k range when there are few rows): the permutation indices of a k chunk
// are loaded once and serve every row, and the rows' gathers are issued
// together.  fp16 input: shift 0, a plain
// gather.  bf16 input: shift puts the row's largest magnitude in
// [2^14, 2^15), so the conversion to fp16 is exact for every value within
// 2^24 of the maximum; the GEMM multiplies the row of y by 2^shift.
constexpr int kXpermRows = 8;  // one warp per row for the row maxima

__global__ void __launch_bounds__(256) xperm_kernel(const XpermParams p) {
    __shared__ int s_shift[kXpermRows];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t m0 = (int64_t)blockIdx.x * kXpermRows;
    const int nrows = (int)min((int64_t)kXpermRows, (int64_t)p.M - m0);
    if (threadIdx.x < kXpermRows) s_shift[threadIdx.x] = 0;
    __syncthreads();
    if (p.x_bf16 && warp < nrows) {
        const uint16_t* row = p.x + (m0 + warp) * p.K;
        int e = 0;
#pragma unroll 8
        for (int k = lane; k < p.K; k += 32) e = max(e, (int)((row[k] >> 7) & 0xFF));
#pragma unroll
        for (int o = 16; o; o >>= 1) e = max(e, __shfl_xor_sync(0xffffffffu, e, o));
        const int shift = (e == 0) ? 0 : e - 141;  // max < 2^(E-126); 2^(E-127-shift) = 2^14
        if (lane == 0) {
            s_shift[warp] = shift;
            if (blockIdx.y == 0) p.xshift[m0 + warp] = shift;
        }
    }
    __syncthreads();
    float f1[kXpermRows], f2[kXpermRows];  // 2^-shift as two normal factors
#pragma unroll
    for (int r = 0; r < kXpermRows; ++r) {
        const int sh = s_shift[r], s1 = sh / 2, s2 = sh - sh / 2;
        f1[r] = __int_as_float((127 - s1) << 23);
        f2[r] = __int_as_float((127 - s2) << 23);
    }
    // k range of this CTA (gridDim.y splits k when there are few rows)
    const int kchunk = ((p.K / 32 + gridDim.y - 1) / gridDim.y) * 32;
    const int kx0 = blockIdx.y * kchunk, kx1 = min(p.K, kx0 + kchunk);
    for (int k0 = kx0 + threadIdx.x * 8; k0 < kx1; k0 += blockDim.x * 8) {
        const int blk = k0 >> 5;
        const int b = p.bits[blk];  // the GEMM refuses a schedule with a bad width
        int idx[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            idx[u] = p.perm[blk * 32 + gemm_code_of_k(b, (k0 & 31) + u)];
            if ((unsigned)idx[u] >= (unsigned)p.K) {
                set_dev_error(QGEMM_DEV_BAD_PERM);
                idx[u] = -1;
            }
        }
#pragma unroll
        for (int r = 0; r < kXpermRows; ++r) {
            if (r >= nrows) break;
            const uint16_t* row = p.x + (m0 + r) * p.K;
            uint32_t h[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const uint32_t raw = idx[u] >= 0 ? (uint32_t)row[idx[u]] : 0u;
                h[u] = p.x_bf16 ? (uint32_t)__half_as_ushort(__float2half_rn(__uint_as_float(raw << 16) * f1[r] * f2[r]))
                                : raw;
            }
            *reinterpret_cast<uint4*>(p.xp + (m0 + r) * p.K + k0) =
                make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16), h[6] | (h[7] << 16));
        }
    }
}

QG_DEV uint32_t h2sub(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
QG_DEV uint32_t h2mul(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// The 32 codes of one block for this thread's column, dequantised to fp16
// pairs in the B tile's order (gemm_code_of_k).  A code at bit k of a half
// (k + b <= 10) becomes 2^(10-k) + q with one mask and an OR of the fp16 of
// 2^(10-k) (0x6400 for 1024 at k = 0, 0x5400 for 64 at k = 4): its mantissa
// step there is 1.  So each pair costs one shift (or funnel shift) of the
// block's words, one mask-and-OR, an exact subtraction of the fp16 of
// 2^(10-k) + z and the multiply by the fp16 scale, the one rounding:
// bit-exact with qgemm_dequant.
// w0 = word row 0 of the block at this column, word rows 1 KB apart.
template <int B>
QG_DEV void dequant_block32(const uint8_t* w0, uint32_t s2, uint32_t (&out)[16]) {
    constexpr uint32_t mask = (1u << B) - 1u;
    uint32_t w[B];
#pragma unroll
    for (int i = 0; i < B; ++i) w[i] = *reinterpret_cast<const uint32_t*>(w0 + i * 1024);
    if constexpr (B == 2 || B == 4 || B == 8) {
        constexpr int per = 16 / B;  // pairs per word
        const uint32_t zoff = 0x64006400u + (((uint32_t)1 << (B - 1)) * 0x00010001u);  // 1024 + z in both halves
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int wi = i / per, sft = (i % per) * B;
            const uint32_t h = lop3_and_or(w[wi] >> sft, mask * 0x00010001u, 0x64006400u);
            out[i] = h2mul(h2sub(h, zoff), s2);
        }
    } else {  // 3, 5, 6: window at stream bit b r - kl (below 0: shifted in zeros)
        constexpr int m = pair_m(B), kl = pair_kl(B), kh = pair_kh(B);
        constexpr uint32_t mlo = kl ? 0x5400u : 0x6400u, mhi = kh ? 0x5400u : 0x6400u;
        constexpr uint32_t pmask = (mask << kl) | (mask << (16 + kh));
        constexpr uint32_t magic = mlo | (mhi << 16);
        constexpr uint32_t z = 1u << (B - 1);
        const uint32_t zpair = (mlo + (z << kl)) | ((mhi + (z << kh)) << 16);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int r = 2 * m * (i / m) + i % m;
            const int base = B * r - kl, end = B * (r + m) + B;  // window start, last bit used + 1
            uint32_t v;
            if (base < 0) {
                v = w[0] << (-base);
            } else {
                const int wi = base >> 5, sh = base & 31;
                if (sh == 0) v = w[wi];
                else if (end <= 32 * (wi + 1)) v = w[wi] >> sh;
                else v = __funnelshift_r(w[wi], w[wi + 1 < B ? wi + 1 : wi], sh);
            }
            out[i] = h2mul(h2sub(lop3_and_or(v, pmask, magic), zpair), s2);
        }
    }
}

QG_DEV void dequant_block32_any(int b, const uint8_t* w0, uint32_t s2, uint32_t (&out)[16]) {
    switch (b) {
        case 2: dequant_block32<2>(w0, s2, out); break;
        case 3: dequant_block32<3>(w0, s2, out); break;
        case 4: dequant_block32<4>(w0, s2, out); break;
        case 5: dequant_block32<5>(w0, s2, out); break;
        case 6: dequant_block32<6>(w0, s2, out); break;
        default: dequant_block32<8>(w0, s2, out); break;
    }
}

// kind::f16 instruction descriptor: fp32 D, A and B both fp16 or both bf16,
// both K-major.
QG_DEV constexpr uint32_t idesc_kf16(int M, int N, bool bf16) {
    return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

template <bool BF16>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const GemmParams p, const __grid_constant__ GemmMaps maps) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nb = p.nb;
    // 1024-byte aligned operand buffers (the swizzle pattern is address based)
    uint8_t* base = smem + ((1024 - (smem_u32(smem) & 1023)) & 1023);
    uint8_t* sA = base;
    uint8_t* sB = sA + kGemmAStages * kGemmABytes;
    uint8_t* sR = sB + kGemmBStages * kGemmBBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sR + kGemmRStages * kGemmRBytes);
    uint64_t* a_full = bars;
    uint64_t* a_empty = a_full + kGemmAStages;
    uint64_t* b_full = a_empty + kGemmAStages;
    uint64_t* b_empty = b_full + kGemmBStages;
    uint64_t* r_full = b_empty + kGemmBStages;
    uint64_t* r_empty = r_full + kGemmRStages;
    uint64_t* acc_full = r_empty + kGemmRStages;
    int* s_misc = reinterpret_cast<int*>(acc_full + 1);  // [0] bad schedule, [1] abort, [2] tmem base
    int32_t* s_offs = s_misc + 8;

    // CTAs below full_tiles take one whole tile each (tile = ntile * mtiles +
    // mt, so neighbours share the weight tile); the rest split the k range of
    // the remaining tiles ksplit ways (neighbours: same k range)
    const int full = p.full_tiles;
    const bool split = (int)blockIdx.x >= full;
    const int rest = p.mtiles * p.ntiles - full;
    const int ks = split ? (int)(blockIdx.x - full) / rest : 0;
    const int tile = split ? full + (int)(blockIdx.x - full) % rest : (int)blockIdx.x;
    const int nsplit = split ? p.ksplit : 1;
    const int mt = tile % p.mtiles, ntile = tile / p.mtiles;
    const int m0 = mt * kGemmBM, n0 = ntile * kGemmBN;
    const int nk_all = (p.K + kGemmBK - 1) / kGemmBK;
    const int kb = (int)((int64_t)ks * nk_all / nsplit);
    const int nk = (int)((int64_t)(ks + 1) * nk_all / nsplit) - kb;  // this CTA's k steps
    const bool two = m0 + 128 < p.M;  // second 128-row half holds rows of x

    // ---- schedule into shared memory, validated before any weight access
    if (tid < 8) s_misc[tid] = 0;
    __syncthreads();
    bool bad = false;
    for (int j = tid; j <= nb; j += kGemmThreads) {
        const int o = p.offs[j];
        s_offs[j] = o;
        if (j < nb) {
            const int b = p.bits[j];
            if (!width_ok(b) || p.offs[j + 1] - o != b) bad = true;
        }
    }
    if (tid == 0 && (p.offs[0] != 0 || (int64_t)p.offs[nb] != p.qw_rows)) bad = true;
    if (bad) atomicOr(&s_misc[0], 1);
    if (tid == 0) {
        for (int i = 0; i < kGemmAStages; ++i) {
            mbar_init(&a_full[i], 1);
            mbar_init(&a_empty[i], 1);
        }
        for (int i = 0; i < kGemmBStages; ++i) {
            mbar_init(&b_full[i], kGemmDecWarps);
            mbar_init(&b_empty[i], 1);
        }
        for (int i = 0; i < kGemmRStages; ++i) {
            mbar_init(&r_full[i], 1);
            mbar_init(&r_empty[i], kGemmDecWarps);
        }
        mbar_init(acc_full, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(reinterpret_cast<uint32_t*>(&s_misc[2]), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = (uint32_t)s_misc[2];
    if (s_misc[0]) {
        if (tid == 0) set_dev_error(QGEMM_DEV_BAD_SCHEDULE);
    } else if (warp == 0) {
        // ================================================= activation producer
        if (lane == 0) {
            const int asub = min(4, (p.M - m0 + 63) / 64);  // 64-row slices of x in this tile
            int i = 0;
            bool ok = true;
            for (; i < nk; ++i) {
                const int sa = i % kGemmAStages;
                if (i >= kGemmAStages && !mbar_wait(&a_empty[sa], (uint32_t)(((i / kGemmAStages) - 1) & 1))) {
                    ok = false;
                    break;
                }
                const int gi = kb + i;  // global k step
                if (asub == 4) {
                    mbar_arrive_expect_tx(&a_full[sa], (uint32_t)kGemmABytes);
                    tma_load_2d(sA + sa * kGemmABytes, &maps.a, gi * kGemmBK, m0, &a_full[sa]);
                } else {
                    // only the 64-row slices that hold rows of x; the MMA also
                    // reads the other rows of the stage, whose accumulator
                    // rows are never stored
                    mbar_arrive_expect_tx(&a_full[sa], (uint32_t)(asub * (kGemmABytes / 4)));
                    for (int q = 0; q < asub; ++q)
                        tma_load_2d(sA + sa * kGemmABytes + q * (kGemmABytes / 4), &maps.a64, gi * kGemmBK,
                                    m0 + 64 * q, &a_full[sa]);
                }
            }
            if (!ok) {  // let every issued copy land before the CTA can exit
                s_misc[1] = 1;
                for (int k = max(0, i - kGemmAStages); k < i; ++k)
                    mbar_wait(&a_full[k % kGemmAStages], (uint32_t)((k / kGemmAStages) & 1));
            }
        }
    } else if (warp == kGemmRawWarp) {
        // ================================================= word-row producer
        // (a warp of its own: its copies do not wait behind the activation
        // tiles' stage releases, nor theirs behind its own)
        if (lane == 0) {
            int i = 0;
            bool ok = true;
            for (; i < nk; ++i) {
                const int sr = i % kGemmRStages;
                if (i >= kGemmRStages && !mbar_wait(&r_empty[sr], (uint32_t)(((i / kGemmRStages) - 1) & 1))) {
                    ok = false;
                    break;
                }
                const int gi = kb + i;  // global k step
                const int j0 = 2 * gi, j1 = min(j0 + 2, nb);
                const int r0 = s_offs[j0], rows = s_offs[j1] - r0;
                const int g = (gi * kGemmBK) / 128;
                const int cols = min(kGemmBN, p.N - n0);
                uint8_t* dst = sR + sr * kGemmRBytes;
                mbar_arrive_expect_tx(&r_full[sr], (uint32_t)(cols * 2 + rows * 1024));
                bulk_g2s(dst, p.scales + (size_t)g * p.N + n0, (uint32_t)cols * 2, &r_full[sr]);
                int r = 0;
#pragma unroll 1
                for (int bx = kGemmBoxMaps - 1; bx >= 0; --bx)
                    if (rows & (1 << bx)) {
                        tma_load_2d(dst + (size_t)(1 + r) * 1024, &maps.w[bx], n0, r0 + r, &r_full[sr]);
                        r += 1 << bx;
                    }
            }
            if (!ok) {  // let every issued copy land before the CTA can exit
                s_misc[1] = 1;
                for (int k = max(0, i - kGemmRStages); k < i; ++k)
                    mbar_wait(&r_full[k % kGemmRStages], (uint32_t)((k / kGemmRStages) & 1));
            }
        }
    } else if (warp == 1) {
        // ================================================= MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdesc = idesc_kf16(128, kGemmBN, BF16);
            for (int i = 0; i < nk && !s_misc[1]; ++i) {
                const int sa = i % kGemmAStages, sb = i % kGemmBStages;
                if (!mbar_wait(&a_full[sa], (uint32_t)((i / kGemmAStages) & 1)) ||
                    !mbar_wait(&b_full[sb], (uint32_t)((i / kGemmBStages) & 1))) {
                    s_misc[1] = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t a_addr = smem_u32(sA + sa * kGemmABytes), b_addr = smem_u32(sB + sb * kGemmBBytes);
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int kk = 0; kk < kGemmBK / 16; ++kk) {
                        if (h == 1 && !two) continue;
                        const uint64_t ad = smem_desc(a_addr + h * (128 * 128) + kk * 32, 16, 1024, 2);
                        const uint64_t bd = smem_desc(b_addr + kk * 32, 16, 1024, 2);
                        tc_mma_ss(tmem + h * kGemmBN, ad, bd, kIdesc, (i | kk) != 0);
                    }
                tc_commit(&a_empty[sa]);
                tc_commit(&b_empty[sb]);
            }
            tc_commit(acc_full);  // also when aborted: completes once issued MMAs are done
        }
    } else {
        // ================================================= dequant warps
        const int n = (tid - 64) & (kGemmBN - 1);  // column within the tile
        const int blk = (tid - 64) >> 8;           // block of the k step (warps 2-9: 0, 10-17: 1)
        for (int i = 0; i < nk; ++i) {
            const int sr = i % kGemmRStages, sb = i % kGemmBStages;
            if (s_misc[1] || !mbar_wait(&r_full[sr], (uint32_t)((i / kGemmRStages) & 1)) ||
                (i >= kGemmBStages && !mbar_wait(&b_empty[sb], (uint32_t)(((i / kGemmBStages) - 1) & 1)))) {
                s_misc[1] = 1;
                break;
            }
            const uint8_t* raw = sR + sr * kGemmRBytes;
            const uint32_t sbits = reinterpret_cast<const uint16_t*>(raw)[n];
            const uint32_t s2 = sbits | (sbits << 16);
            uint8_t* brow = sB + sb * kGemmBBytes + n * 128;
            const int j0 = 2 * (kb + i);
            const int r0 = s_offs[j0];
            {
                const int j = j0 + blk;
                uint32_t out[16];
                if (j < nb) {
                    dequant_block32_any(s_offs[j + 1] - s_offs[j],
                                        raw + 1024 + (size_t)(s_offs[j] - r0) * 1024 + n * 4, s2, out);
                } else {
#pragma unroll
                    for (int u = 0; u < 16; ++u) out[u] = 0;
                }
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int chunk = 4 * blk + c;
                    *reinterpret_cast<uint4*>(brow + ((chunk ^ (n & 7)) << 4)) =
                        make_uint4(out[4 * c], out[4 * c + 1], out[4 * c + 2], out[4 * c + 3]);
                }
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&b_full[sb]);
                mbar_arrive(&r_empty[sr]);
            }
        }
        // ---- epilogue: TMEM -> y (fp16), or fp32 partial sums under split K
        const bool ok = mbar_wait(acc_full, 0) && !s_misc[1];
        tc_fence_after();
        // warp: TMEM lane quadrant warp % 4 (the only lanes it may access),
        // accumulator (128-row half) h and 128-column half ch
        const int q = warp & 3, sel = (warp - 2) >> 2, h = sel & 1, ch = sel >> 1;
        const int rl = h * 128 + q * 32 + lane;  // row within the tile
        const int row = m0 + rl;
        const int sh = (p.x_bf16 && row < p.M) ? p.xshift[row] : 0;
        const float g1 = __int_as_float((127 + sh / 2) << 23), g2 = __int_as_float((127 + (sh - sh / 2)) << 23);
        auto store_y = [&](int r, int c, const float (&v)[16], float s1, float s2) {
            uint32_t hv[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const __half2 t = __floats2half2_rn(v[2 * u] * s1 * s2, v[2 * u + 1] * s1 * s2);
                hv[u] = *reinterpret_cast<const uint32_t*>(&t);
            }
            __half* dst = p.y + (size_t)r * p.N + n0 + c;
            *reinterpret_cast<uint4*>(dst) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
            if (n0 + c + 8 < p.N) *reinterpret_cast<uint4*>(dst + 8) = make_uint4(hv[4], hv[5], hv[6], hv[7]);
        };
        if (ok && (h == 0 || two)) {
            const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + h * kGemmBN;
            float* part =
                p.partial + ((size_t)(tile - full) * nsplit + ks) * (kGemmBM * kGemmBN) + (size_t)rl * kGemmBN;
#pragma unroll 1
            for (int c = ch * (kGemmBN / 2); c < (ch + 1) * (kGemmBN / 2); c += 16) {
                float v[16];
                tmem_ld16(taddr + c, v);
                if (nsplit == 1) {
                    if (row < p.M && n0 + c < p.N) store_y(row, c, v, g1, g2);
                } else if (row < p.M) {  // the reduction reads the tile's rows of x only
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        __stcg(reinterpret_cast<float4*>(part + c + 4 * u),
                               make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]));
                }
            }
        }
        if (nsplit > 1) {
            // the last of the tile's nsplit CTAs adds the partial sums in split
            // order (the same bits on every call), one float4 per thread step
            __threadfence();
            named_bar_sync(1, kGemmDecWarps * 32);
            if (tid == 64) s_misc[3] = (ok && !s_misc[1]) ? (atomicAdd(&p.tickets[tile], 1) == nsplit - 1) : 0;
            named_bar_sync(1, kGemmDecWarps * 32);
            if (s_misc[3]) {
                __threadfence();
                const float4* base4 =
                    reinterpret_cast<const float4*>(p.partial + (size_t)(tile - full) * nsplit * (kGemmBM * kGemmBN));
                const int t = tid - 64;
                const int rows = min(kGemmBM, p.M - m0);
#pragma unroll 2
                for (int f = t; f < rows * (kGemmBN / 4); f += kGemmDecWarps * 32) {
                    const int r2 = f / (kGemmBN / 4), c4 = (f % (kGemmBN / 4)) * 4;
                    if (n0 + c4 >= p.N) continue;
                    float4 a[kGemmMaxSplit];
#pragma unroll
                    for (int kq = 0; kq < kGemmMaxSplit; ++kq)
                        if (kq < nsplit) a[kq] = __ldcg(base4 + (size_t)kq * (kGemmBM * kGemmBN / 4) + f);
                    float4 sum = a[0];
#pragma unroll
                    for (int kq = 1; kq < kGemmMaxSplit; ++kq)
                        if (kq < nsplit) {
                            sum.x += a[kq].x;
                            sum.y += a[kq].y;
                            sum.z += a[kq].z;
                            sum.w += a[kq].w;
                        }
                    const int row2 = m0 + r2;
                    const int sh2 = p.x_bf16 ? p.xshift[row2] : 0;
                    const float s1 = __int_as_float((127 + sh2 / 2) << 23);
                    const float s2 = __int_as_float((127 + (sh2 - sh2 / 2)) << 23);
                    const __half2 lo = __floats2half2_rn(sum.x * s1 * s2, sum.y * s1 * s2);
                    const __half2 hi = __floats2half2_rn(sum.z * s1 * s2, sum.w * s1 * s2);
                    *reinterpret_cast<uint2*>(p.y + (size_t)row2 * p.N + n0 + c4) =
                        make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
                }
                if (tid == 64) p.tickets[tile] = 0;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace qg
