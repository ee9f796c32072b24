// Integer split-K GEMV for decode with M <= 4 tokens: y = x[:, perm] . dequant(Wq).
//
// At M = 1 the decode kernel must consume about 85 codes per clock per SM to
// stream 2.55-bit weights at B200's HBM bandwidth, so the arithmetic per code
// decides the speed.  Tensor cores cannot help at this batch size: expanding
// the codes to 16-bit operands in TMEM or shared memory needs more on-chip
// bandwidth than B200 has, and the legacy warp MMA is not native on sm_100.
// This kernel instead uses the integer dot-product instruction dp2a
// (2 x int16 * 2 x uint8 + int32), native on sm_100:
//
// * xprep_int_kernel quantises the gathered activations per (128-row group,
//   token) to int16 with a power-of-two scale 2^e chosen so that the group's
//   largest magnitude maps to at most 2^14 (a group's int32 sum of 128
//   products then cannot overflow), in the order in which the decoder below
//   consumes codes, and stores per (block, token) z * sum(x_int): the zero
//   point's share.  Error: at most half a unit of 2^-e per activation.  A
//   block whose group holds an activation far larger than the block's other
//   ones (an outlier channel) would lose those others to that rounding, even
//   where the outlier's own weight row is zero; such a block also gets the
//   rounding residue as a second int16 part on a grid 2^15 times finer, and
//   the decoder runs its dot products twice.
// * gemv_int_kernel moves codes into bytes with one shift and one mask per
//   four codes (2- and 4-bit widths; odd widths need a few more), and
//   accumulates sum_k x_int * q exactly in int32 with dp2a, starting from
//   -z * sum(x_int); each group's integer sum is then converted once and
//   multiplied by the (group, column) scale and 2^-e in fp32.
//
// Work split as in gemv.cuh, with units of (256-column tile, two 128-row
// groups) = 8 blocks: the units of all tiles are cut into one contiguous range
// per CTA (two CTAs per SM for M <= 2, one for M <= 4) of equal cost (word
// rows plus one per unit).  Two copy warps stream each unit into a
// shared-memory ring of 1 KB rows: its word rows (2D tensor copies of 2^i rows
// x 256 columns, one per set bit of the row count), its scale rows (bulk
// copies) and its activation records (a bulk copy, from a warp of its own:
// weights are issued before the wait for the activation kernel, records after
// it).  Consumer warps 0-7: warp w decodes block w/2 of each group of the unit
// for the 128 columns of half w%2, four adjacent columns per thread (one
// 16-byte load per word row); the four block slots are added in shared memory
// when a tile is done.  A tile shared with other CTAs leaves a partial sum in
// the workspace; the tickets that pick the CTA which adds them up are taken
// once, after the CTA's last unit, so no cross-CTA round trip stalls the
// stream.
#pragma once

#include <cuda.h>

#include "gemv.cuh"

namespace qg {

constexpr int kIntMaxM = 4;
constexpr int kIntThreads = kGemvDecThreads + 64;  // 8 consumer warps, 2 copy warps
constexpr int kIntRowBytes = 1024;   // one ring row: 256 words (a box row lands densely)
constexpr int kIntBoxMaps = 7;       // tensor maps with box heights 1, 2, 4, ..., 64 rows
constexpr int kIntUnitGroups = 2;    // 128-row groups per unit
constexpr int kIntUnitBlocks = kIntUnitGroups * kGemvGroupBlocks;  // 8 blocks, 256 rows

// Tensor maps over qw [qw_rows][N] uint32, box {256 columns, 2^i rows}.
struct IntMaps {
    CUtensorMap box[kIntBoxMaps];
};

// Ring rows of a unit: one row holding its two scale rows (512 B each), the
// word rows, the activation records.
__host__ __device__ constexpr int int_unit_rows(int wrows, int nblk, int rec_bytes) {
    return 1 + wrows + (nblk * rec_bytes + kIntRowBytes - 1) / kIntRowBytes;
}

// Bytes of one block's activation record: int16 x_hi[MP][32] and
// x_lo[MP][32] in decoder order, int32 zsum_hi[MP], zsum_lo[MP], e[MP], and
// one int32 flag (the low part is used); padded to 16 bytes.
__host__ __device__ constexpr int int_rec_bytes(int mp) { return (140 * mp + 4 + 15) / 16 * 16; }
__host__ __device__ constexpr int int_rec_zhi(int mp) { return 128 * mp; }
__host__ __device__ constexpr int int_rec_zlo(int mp) { return 132 * mp; }
__host__ __device__ constexpr int int_rec_e(int mp) { return 136 * mp; }
__host__ __device__ constexpr int int_rec_flag(int mp) { return 140 * mp; }

// A block needs the low part when its group's largest scaled magnitude gmax
// exceeds twice the root sum of squares of the block's activations other than
// its largest one: the first part's rounding error (at most 2^-15 gmax per
// activation) then stays below 2^-12 of what those activations contribute.
QG_DEV bool int_needs_low(float gmax, float block_sq, float block_max) {
    const float rest = block_sq - block_max * block_max;
    return gmax * gmax > 4.f * fmaxf(rest, 0.f);
}

struct IntPrepParams {
    const void* x;
    const int32_t* perm;
    const uint8_t* bits;
    uint8_t* rec;   // [nb][int_rec_bytes(mp)]
    int M, K, nb, mp, x_bf16;
};

struct IntParams {
    const uint8_t* rec;
    const uint32_t* qw;
    int64_t qw_rows;
    const __half* scales;
    const uint8_t* bits;
    const int32_t* offs;
    __half* y;
    int* tickets;   // [tiles]
    float* slots;   // [gridDim.x][2][MP][256]
    int M, K, N, nb, ng, tiles;
    int ring_rows;
};

// Code index (within the block) that the dp2a decoder pairs with activation
// position k (pair k/2, half k%2).
QG_DEV int int_code_of_k(int b, int k) {
    const int j = k >> 1, h = k & 1;
    if (b == 2) return 16 * (j >> 3) + ((j & 7) >> 1) + 8 * (j & 1) + 4 * h;
    if (b == 4) return 8 * (j >> 2) + ((j & 3) >> 1) + 4 * (j & 1) + 2 * h;
    return k;  // 3, 5, 6, 8: bytes in natural order
}

QG_DEV int32_t dp2a_lo(uint32_t xpair, uint32_t bytes, int32_t c) {
    int32_t d;
    asm("dp2a.lo.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(xpair), "r"(bytes), "r"(c));
    return d;
}
QG_DEV int32_t dp2a_hi(uint32_t xpair, uint32_t bytes, int32_t c) {
    int32_t d;
    asm("dp2a.hi.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(xpair), "r"(bytes), "r"(c));
    return d;
}

// Four B-bit fields at bits 0, B, 2B, 3B of X, one per byte.
template <int B>
QG_DEV uint32_t spread4(uint32_t X) {
    constexpr uint32_t m = (1u << B) - 1u;
    return (X & m) | ((X << (8 - B)) & (m << 8)) | ((X << (16 - 2 * B)) & (m << 16)) |
           ((X << (24 - 3 * B)) & (m << 24));
}

QG_DEV uint32_t comp(const uint4& v, int q) { return q == 0 ? v.x : q == 1 ? v.y : q == 2 ? v.z : v.w; }

// acc is scaled by 2^int_acc_shift(B): 2- and 4-bit codes are used in place
// (masked, not shifted down), so a code at bit offset 2s of its byte enters as
// q * 4^s; Horner steps between the offsets bring every term to the same
// power of two, exactly.
QG_DEV constexpr int int_acc_shift(int b) { return b == 2 ? 6 : b == 4 ? 4 : 0; }

// One block of width B for the thread's 4 adjacent columns:
// acc[q][t] = 2^int_acc_shift(B) * (acc[q][t] + sum_k x_int[t][k] * code[k][col q]).
// v[i] = word row i of the block at the thread's 4 columns.
template <int B, int MP>
QG_DEV void block_dp2a_v(const uint4 (&v)[B], const uint32_t (&xp)[MP][16], int32_t (&acc)[4][MP]) {
    if constexpr (B == 2) {
        // word wi, byte i: codes 16wi+4i+s at bits 2s; mask s keeps q * 4^s
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const uint32_t mask = 0x03030303u << (2 * s);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint32_t m0 = comp(v[0], q) & mask, m1 = comp(v[1], q) & mask;
#pragma unroll
                for (int t = 0; t < MP; ++t) {
                    int32_t a = (s == 0) ? acc[q][t] : acc[q][t] * 4;
                    a = dp2a_lo(xp[t][2 * s], m0, a);
                    a = dp2a_hi(xp[t][2 * s + 1], m0, a);
                    a = dp2a_lo(xp[t][8 + 2 * s], m1, a);
                    acc[q][t] = dp2a_hi(xp[t][8 + 2 * s + 1], m1, a);
                }
            }
        }
    } else if constexpr (B == 4) {
        // word wi: low nibbles of its bytes are codes 8wi+2i, high nibbles 8wi+2i+1 (as 16 q)
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int t = 0; t < MP; ++t) {
                int32_t a = acc[q][t];
#pragma unroll
                for (int wi = 0; wi < 4; ++wi) {
                    const uint32_t e = comp(v[wi], q) & 0x0F0F0F0Fu;
                    a = dp2a_lo(xp[t][4 * wi + 0], e, a);
                    a = dp2a_hi(xp[t][4 * wi + 1], e, a);
                }
                a *= 16;
#pragma unroll
                for (int wi = 0; wi < 4; ++wi) {
                    const uint32_t o = comp(v[wi], q) & 0xF0F0F0F0u;
                    a = dp2a_lo(xp[t][4 * wi + 2], o, a);
                    a = dp2a_hi(xp[t][4 * wi + 3], o, a);
                }
                acc[q][t] = a;
            }
    } else if constexpr (B == 8) {
#pragma unroll
        for (int wi = 0; wi < 8; ++wi) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int t = 0; t < MP; ++t) {
                    acc[q][t] = dp2a_lo(xp[t][2 * wi], comp(v[wi], q), acc[q][t]);
                    acc[q][t] = dp2a_hi(xp[t][2 * wi + 1], comp(v[wi], q), acc[q][t]);
                }
        }
    } else {  // 3, 5, 6: codes 4c..4c+3 from a window at bit 4cB, spread into bytes
#pragma unroll
        for (int q = 0; q < 4; ++q) {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const int bit = 4 * c * B, wi = bit >> 5, sh = bit & 31;
                // a window never ends past the last word: 4 * 8 * B = 32 * B bits
                const uint32_t X = (sh + 4 * B <= 32)
                                       ? comp(v[wi], q) >> sh
                                       : __funnelshift_r(comp(v[wi], q), comp(v[wi + 1 < B ? wi + 1 : wi], q), sh);
                const uint32_t by = spread4<B>(X);
#pragma unroll
                for (int t = 0; t < MP; ++t) {
                    acc[q][t] = dp2a_lo(xp[t][2 * c], by, acc[q][t]);
                    acc[q][t] = dp2a_hi(xp[t][2 * c + 1], by, acc[q][t]);
                }
            }
        }
    }
}

// The same, reading the block's word rows from the shared-memory ring (rows
// kIntRowBytes apart).  w = word row 0 of the block at the thread's first column.
template <int B, int MP>
QG_DEV void block_dp2a(const uint8_t* w, const uint32_t (&xp)[MP][16], int32_t (&acc)[4][MP]) {
    uint4 v[B];
#pragma unroll
    for (int i = 0; i < B; ++i) v[i] = *reinterpret_cast<const uint4*>(w + i * kIntRowBytes);
    block_dp2a_v<B, MP>(v, xp, acc);
}

// ------------------------------------------------------------------ xprep
// One warp per block (lane = position in the decoder's order), 8 blocks = 2
// groups per CTA.  Group maximum -> e; x_int = rint(x * 2^e); zsum =
// z * sum of the block's x_int.
__global__ void __launch_bounds__(256) xprep_int_kernel(const IntPrepParams p) {
    // launched as a programmatic dependent of the previous grid in the stream
    // (a decode GEMV, say): x may be that grid's output and the records below
    // may still be read by it, so wait for it before any load of x or store
    asm volatile("griddepcontrol.launch_dependents;");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    __shared__ int s_gmax[2][kIntMaxM];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gl = warp >> 2;
    if (threadIdx.x < 2 * kIntMaxM) s_gmax[threadIdx.x / kIntMaxM][threadIdx.x % kIntMaxM] = 0;
    const int j = blockIdx.x * 8 + warp;
    const int b = (j < p.nb) ? (int)p.bits[j] : 2;
    const bool live = (j < p.nb) && width_ok(b);
    if (j < p.nb && !width_ok(b) && lane == 0) set_dev_error(QGEMM_DEV_BAD_SCHEDULE);
    int src = 0;
    if (live) {
        src = p.perm[j * kBlockRows + int_code_of_k(b, lane)];
        if (src < 0 || src >= p.K) {
            set_dev_error(QGEMM_DEV_BAD_PERM);
            src = 0;
        }
    }
    float v[kIntMaxM];
#pragma unroll
    for (int m = 0; m < kIntMaxM; ++m) {
        v[m] = 0.f;
        if (live && m < p.M) {
            const uint16_t raw = reinterpret_cast<const uint16_t*>(p.x)[(size_t)m * p.K + src];
            v[m] = p.x_bf16 ? __uint_as_float((uint32_t)raw << 16) : __half2float(__ushort_as_half(raw));
        }
    }
    __syncthreads();
#pragma unroll
    for (int m = 0; m < kIntMaxM; ++m) {
        if (m >= p.M) break;  // uniform over the block
        int a = __float_as_int(fabsf(v[m]));
        if (a >= 0x7F800000) a = 0x7F7FFFFF;  // inf / nan: saturate the scale choice
#pragma unroll
        for (int o = 16; o; o >>= 1) a = max(a, __shfl_xor_sync(0xffffffffu, a, o));
        if (lane == 0) atomicMax(&s_gmax[gl][m], a);
    }
    __syncthreads();
    if (j >= p.nb) return;
    const int rb = int_rec_bytes(p.mp);
    uint8_t* rec = p.rec + (size_t)j * rb;
    const int z = 1 << (b - 1);
    bool low = false;
#pragma unroll
    for (int m = 0; m < kIntMaxM; ++m) {
        if (m >= p.mp) break;  // uniform over the block
        int e = 0, xi = 0, xl = 0;
        if (m < p.M && m < kIntMaxM) {
            const int E = (s_gmax[gl][m] >> 23) & 0xFF;  // max < 2^(E - 126)
            e = (E == 0) ? 140 : 140 - E;
            const int e1 = e / 2, e2 = e - e / 2;
            const float p1 = __int_as_float((127 + e1) << 23), p2 = __int_as_float((127 + e2) << 23);
            const float f = v[m] * p1 * p2;  // exact: a power-of-two scaling
            if (live) {
                xi = __float2int_rn(f);
                // f - xi is exact (|f| < 2^15) and at most 1/2; its int16 part
                // on a grid of 2^-15 leaves at most 2^-16
                xl = __float2int_rn((f - (float)xi) * 32768.f);
            }
            // outlier test in the scaled domain (all magnitudes below 2^15)
            const float gmax = __int_as_float(s_gmax[gl][m]) * p1 * p2;
            float sq = f * f, bm = fabsf(f);
#pragma unroll
            for (int o = 16; o; o >>= 1) {
                sq += __shfl_xor_sync(0xffffffffu, sq, o);
                bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
            }
            low = low || int_needs_low(gmax, sq, bm);
        }
        reinterpret_cast<int16_t*>(rec)[m * 32 + lane] = (int16_t)xi;
        reinterpret_cast<int16_t*>(rec)[(p.mp + m) * 32 + lane] = (int16_t)xl;
        int sum = xi, suml = xl;
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            sum += __shfl_xor_sync(0xffffffffu, sum, o);
            suml += __shfl_xor_sync(0xffffffffu, suml, o);
        }
        if (lane == 0) {
            reinterpret_cast<int32_t*>(rec + int_rec_zhi(p.mp))[m] = z * sum;
            reinterpret_cast<int32_t*>(rec + int_rec_zlo(p.mp))[m] = z * suml;
            reinterpret_cast<int32_t*>(rec + int_rec_e(p.mp))[m] = e;
        }
    }
    if (lane == 0) *reinterpret_cast<int32_t*>(rec + int_rec_flag(p.mp)) = low ? 1 : 0;
}

// -------------------------------------------------------------------- GEMV
template <int MP>
__global__ void __launch_bounds__(kIntThreads, MP <= 2 ? 2 : 1)
    gemv_int_kernel(const IntParams p, const __grid_constant__ IntMaps maps) {
    constexpr int REC = int_rec_bytes(MP);
    constexpr int TP = MP < 4 ? MP : 4;  // tokens per pass
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nb = p.nb, ng = p.ng, M = p.M;
    // the next call's activation kernel may start during this grid's tail; it
    // waits for this grid's completion before it touches x or the workspace
    if (tid == 0) asm volatile("griddepcontrol.launch_dependents;");

    int32_t* s_offs = reinterpret_cast<int32_t*>(smem);
    size_t o = ((size_t)(nb + 1) * 4 + 15) & ~(size_t)15;
    uint64_t* s_full = reinterpret_cast<uint64_t*>(smem + o);
    o += kGemvSlots * 8;
    uint64_t* s_empty = reinterpret_cast<uint64_t*>(smem + o);
    o += kGemvSlots * 8;
    int* s_misc = reinterpret_cast<int*>(smem + o);  // bad schedule, last flags (2), abort
    o += 64;
    float* s_red = reinterpret_cast<float*>(smem + o);  // [3][256][MP] block slots 1..3
    o += (size_t)3 * kGemvTileCols * MP * 4;
    o = (o + 1023) & ~(size_t)1023;
    uint8_t* s_ring = smem + o;
    const int R = p.ring_rows;

    // ---- schedule into shared memory (one round trip), validated
    if (tid < 16) s_misc[tid] = 0;
    int32_t my_off[4], my_next[4];
    uint8_t my_bits[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int j = tid + q * kIntThreads;
        my_off[q] = (j <= nb) ? p.offs[j] : 0;
        my_next[q] = (j < nb) ? p.offs[j + 1] : 0;
        my_bits[q] = (j < nb) ? p.bits[j] : (uint8_t)2;
    }
    for (int j = tid + 4 * kIntThreads; j <= nb; j += kIntThreads) s_offs[j] = p.offs[j];
    bool bad = false;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int j = tid + q * kIntThreads;
        if (j <= nb) s_offs[j] = my_off[q];
        if (j < nb && (!width_ok(my_bits[q]) || my_next[q] - my_off[q] != my_bits[q])) bad = true;
    }
    for (int j = tid + 4 * kIntThreads; j < nb; j += kIntThreads) {
        const int b = p.bits[j];
        if (!width_ok(b) || p.offs[j + 1] - p.offs[j] != b) bad = true;
    }
    if (tid == 0 && (my_off[0] != 0 || (int64_t)p.offs[nb] != p.qw_rows)) bad = true;
    __syncthreads();
    if (bad) atomicOr(&s_misc[0], 1);
    if (tid == 0) {
        for (int i = 0; i < kGemvSlots; ++i) {
            mbar_init(&s_full[i], 3);  // the three issuers of the copy warps
            mbar_init(&s_empty[i], kGemvDecWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();
    if (s_misc[0]) {
        if (tid == 0) {
            set_dev_error(QGEMM_DEV_BAD_SCHEDULE);
            asm volatile("griddepcontrol.wait;" ::: "memory");
        }
        return;
    }
    // units: (tile, pair of groups) = 8 blocks; nu units per tile
    const int nu = (nb + kIntUnitBlocks - 1) / kIntUnitBlocks;
    const int64_t W = s_offs[nb];
    const int64_t C = (int64_t)p.tiles * (W + nu);
    const int64_t G = gridDim.x;
    const int64_t u0 = unit_start(blockIdx.x, G, C, W, nb, nu, p.tiles, s_offs, kIntUnitBlocks);
    const int64_t u1 = unit_start(blockIdx.x + 1, G, C, W, nb, nu, p.tiles, s_offs, kIntUnitBlocks);
    const int nunits = (int)(u1 - u0);
    if (nunits <= 0) {
        if (tid == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
        return;
    }
    const int t0 = (int)(u0 / nu), gf = (int)(u0 - (int64_t)t0 * nu);
    auto rows_of = [&](int gg) {
        const int a = gg * kIntUnitBlocks, bb = min(a + kIntUnitBlocks, nb);
        return int_unit_rows(s_offs[bb] - s_offs[a], bb - a, REC);
    };

    // =================================================== producer warps
    // Three issuers split each unit's copies: lane 0 of warp 8 the word rows
    // (2D boxes), lane 1 of warp 8 the scale rows, lane 0 of warp 9 the
    // activation records.  A copy instruction can wait for room in the SM's
    // copy queue, so the records, which the activation kernel may only just
    // have written, get a warp of their own and are not held behind the
    // weights that the other lanes issue ahead of them.  Every issuer takes the
    // same ring positions and the same waits, in the same order, so they issue
    // the same units; lanes 0 and 1 of warp 8 agree on every wait's outcome.
    if (warp >= kGemvDecWarps) {
        const int role = (warp == kGemvDecWarps) ? (lane < 2 ? lane : 3) : (lane == 0 ? 2 : 3);
        if (role > 2) return;
        const unsigned peers = (role == 2) ? 0x1u : 0x3u;
        auto issue = [&](int k, int t, int g, int row) {
            const int j0 = g * kIntUnitBlocks, j1 = min(j0 + kIntUnitBlocks, nb);
            const int r0 = s_offs[j0], wrows = s_offs[j1] - r0;
            uint64_t* bar = &s_full[k & (kGemvSlots - 1)];
            uint8_t* dst = s_ring + (size_t)row * kIntRowBytes;
            if (role == 0) {
                mbar_arrive_expect_tx(bar, (uint32_t)(wrows * kIntRowBytes));
                int r = 0;
#pragma unroll 1
                for (int i = kIntBoxMaps - 1; i >= 0; --i)
                    if (wrows & (1 << i)) {
                        tma_load_2d(dst + (size_t)(1 + r) * kIntRowBytes, &maps.box[i], t * kGemvTileCols, r0 + r,
                                    bar);
                        r += 1 << i;
                    }
            } else if (role == 1) {
                const int cols = min(kGemvTileCols, p.N - t * kGemvTileCols);
                const int g0 = g * kIntUnitGroups, ngr = min(kIntUnitGroups, ng - g0);
                mbar_arrive_expect_tx(bar, (uint32_t)(ngr * cols * 2));
                for (int u = 0; u < ngr; ++u)
                    bulk_g2s(dst + u * 512, p.scales + (size_t)(g0 + u) * p.N + (size_t)t * kGemvTileCols,
                             (uint32_t)cols * 2, bar);
            } else {
                const int nblk = j1 - j0;
                mbar_arrive_expect_tx(bar, (uint32_t)(nblk * REC));
                bulk_g2s(dst + (size_t)(1 + wrows) * kIntRowBytes, p.rec + (size_t)j0 * REC, (uint32_t)nblk * REC,
                         bar);
            }
        };
        // Units that fit the ring and the slots before any release; the
        // records issuer first waits for the activation kernel.
        int npre = 0;
        {
            int pp = 0, gg = gf;
            int64_t tot = 0;
            while (npre < nunits && npre < kGemvSlots) {
                int p2 = pp;
                int64_t t2 = tot;
                ring_alloc(p2, t2, rows_of(gg), R);
                if (t2 > R) break;
                pp = p2;
                tot = t2;
                ++npre;
                if (++gg == nu) gg = 0;
            }
        }
        if (role == 2) asm volatile("griddepcontrol.wait;" ::: "memory");  // records come from xprep_int
        int pos = 0;
        int64_t total = 0;
        int t = t0, g = gf;
        for (int k = 0; k < npre; ++k) {
            issue(k, t, g, ring_alloc(pos, total, rows_of(g), R));
            if (++g == nu) { g = 0; ++t; }
        }
        int pos_rel = 0;
        int64_t total_rel = 0;
        int k_rel = 0, g_rel = gf;
        bool ok = true;
        int k = npre;
        for (; k < nunits; ++k) {
            const int need = rows_of(g);
            int ppos = pos;
            int64_t ptotal = total;
            ring_alloc(ppos, ptotal, need, R);
            // room: the unit's rows are free once everything allocated more
            // than R rows earlier is released; an empty ring (k_rel == k) always
            // has room, which also covers a unit whose skipped tail plus its own
            // rows exceed R
            while (k - k_rel >= kGemvSlots || (ptotal - total_rel > R && k_rel < k)) {
                const bool w = mbar_wait(&s_empty[k_rel & (kGemvSlots - 1)], (uint32_t)((k_rel / kGemvSlots) & 1));
                if (!__all_sync(peers, w)) {
                    ok = false;
                    break;
                }
                ring_alloc(pos_rel, total_rel, rows_of(g_rel), R);
                ++k_rel;
                if (++g_rel == nu) g_rel = 0;
            }
            if (!ok) break;
            issue(k, t, g, ring_alloc(pos, total, need, R));
            if (++g == nu) { g = 0; ++t; }
        }
        if (!ok) {
            // let this issuer's copies in flight land before the CTA can exit
            s_misc[3] = 1;
            for (int kk = k_rel; kk < k; ++kk)
                if (!mbar_wait(&s_full[kk & (kGemvSlots - 1)], (uint32_t)((kk / kGemvSlots) & 1))) break;
        }
        return;
    }

    // =================================================== consumer warps 0-7
    const int bi = warp >> 1;                 // block slot within each group of the unit
    const int col0 = (warp & 1) * 128 + lane * 4;
    float yacc[4][MP];
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int t = 0; t < MP; ++t) yacc[q][t] = 0.f;
    bool aborted = false;
    int pend0 = -1, pend1 = -1;  // shared first / last tile: partial sums wait for a ticket

    // Tile done: add the four block slots (slots 1..3 through shared memory),
    // then write y, or the partial sum when other CTAs share the tile.
    auto flush = [&](int tt) {
        if (bi > 0) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int t = 0; t < MP; ++t) s_red[((bi - 1) * kGemvTileCols + col0 + q) * MP + t] = yacc[q][t];
        }
        named_bar_sync(1, kGemvDecThreads);
        const int64_t ut0 = (int64_t)tt * nu;
        const int first = cta_of(ut0, G, C, W, nu, s_offs, kIntUnitBlocks);
        const int last = cta_of(ut0 + nu - 1, G, C, W, nu, s_offs, kIntUnitBlocks);
        const int ncol = p.N - tt * kGemvTileCols;
        if (bi == 0) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int t = 0; t < MP; ++t)
                    yacc[q][t] += s_red[(col0 + q) * MP + t] + s_red[(kGemvTileCols + col0 + q) * MP + t] +
                                  s_red[(2 * kGemvTileCols + col0 + q) * MP + t];
            if (first == last) {
                if (!aborted)
#pragma unroll
                    for (int q = 0; q < 4; ++q)
#pragma unroll
                        for (int t = 0; t < MP; ++t)
                            if (t < M && col0 + q < ncol)
                                p.y[(size_t)t * p.N + (size_t)tt * kGemvTileCols + col0 + q] =
                                    __float2half_rn(yacc[q][t]);
            } else {
                const int which = (u0 < ut0) ? 1 : 0;
                float* my = p.slots + ((size_t)blockIdx.x * 2 + which) * (MP * kGemvTileCols);
#pragma unroll
                for (int t = 0; t < MP; ++t)
                    if (t < M)
                        *reinterpret_cast<float4*>(my + t * kGemvTileCols + col0) =
                            make_float4(yacc[0][t], yacc[1][t], yacc[2][t], yacc[3][t]);
            }
        }
        if (first != last) {
            if (u0 < ut0) pend1 = tt;
            else pend0 = tt;
        }
        named_bar_sync(1, kGemvDecThreads);
    };

    int pos = 0;
    int64_t total = 0;
    int t = t0, g = gf, t_prev = t0;
    for (int k = 0; k < nunits; ++k) {
        if (t != t_prev) {
            flush(t_prev);
            t_prev = t;
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int tt = 0; tt < MP; ++tt) yacc[q][tt] = 0.f;
        }
        const int j0 = g * kIntUnitBlocks, j1 = min(j0 + kIntUnitBlocks, nb);
        const int o0 = s_offs[j0];
        const int wrows = s_offs[j1] - o0;
        const int row = ring_alloc(pos, total, int_unit_rows(wrows, j1 - j0, REC), R);
        const int slot = k & (kGemvSlots - 1);
        if (!aborted && (s_misc[3] || !mbar_wait(&s_full[slot], (uint32_t)((k / kGemvSlots) & 1)))) {
            aborted = true;
            s_misc[3] = 1;
        }
        const uint8_t* ub = s_ring + (size_t)row * kIntRowBytes;
#pragma unroll 1
        for (int gi = 0; gi < kIntUnitGroups; ++gi) {
            const int bs = gi * kGemvGroupBlocks + bi;  // block slot within the unit
            const int j = j0 + bs;
            if (aborted || j >= j1) continue;
            const int b = s_offs[j + 1] - s_offs[j];
            const uint8_t* rec = ub + (size_t)(1 + wrows) * kIntRowBytes + bs * REC;
            const uint8_t* wb = ub + (size_t)(1 + s_offs[j] - o0) * kIntRowBytes + col0 * 4;
            const uint2 sv = *reinterpret_cast<const uint2*>(ub + gi * 512 + col0 * 2);
            float sc[4];
            sc[0] = __low2float(*reinterpret_cast<const __half2*>(&sv.x));
            sc[1] = __high2float(*reinterpret_cast<const __half2*>(&sv.x));
            sc[2] = __low2float(*reinterpret_cast<const __half2*>(&sv.y));
            sc[3] = __high2float(*reinterpret_cast<const __half2*>(&sv.y));
            // tokens in passes of up to four (registers); each pass re-reads the
            // block's word rows from shared memory, once per activation part
            const int nparts = 1 + *reinterpret_cast<const int32_t*>(rec + int_rec_flag(MP));
#pragma unroll
            for (int ps = 0; ps < MP / TP; ++ps) {
#pragma unroll 1
                for (int part = 0; part < nparts; ++part) {
                    uint32_t xp[TP][16];
                    int32_t acc[4][TP];
#pragma unroll
                    for (int tt = 0; tt < TP; ++tt) {
                        const uint4* xr = reinterpret_cast<const uint4*>(rec + (part * MP + ps * TP + tt) * 64);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const uint4 v = xr[i];
                            xp[tt][4 * i] = v.x;
                            xp[tt][4 * i + 1] = v.y;
                            xp[tt][4 * i + 2] = v.z;
                            xp[tt][4 * i + 3] = v.w;
                        }
                        const int32_t zs =
                            reinterpret_cast<const int32_t*>(rec + (part ? int_rec_zlo(MP) : int_rec_zhi(MP)))[ps * TP + tt];
#pragma unroll
                        for (int q = 0; q < 4; ++q) acc[q][tt] = -zs;
                    }
                    switch (b) {
                        case 2: block_dp2a<2, TP>(wb, xp, acc); break;
                        case 3: block_dp2a<3, TP>(wb, xp, acc); break;
                        case 4: block_dp2a<4, TP>(wb, xp, acc); break;
                        case 5: block_dp2a<5, TP>(wb, xp, acc); break;
                        case 6: block_dp2a<6, TP>(wb, xp, acc); break;
                        default: block_dp2a<8, TP>(wb, xp, acc); break;
                    }
                    // the low part's grid is 2^-15 of the high part's
#pragma unroll
                    for (int tt = 0; tt < TP; ++tt) {
                        const int e = reinterpret_cast<const int32_t*>(rec + int_rec_e(MP))[ps * TP + tt] +
                                      int_acc_shift(b) + 15 * part;
                        const int e1 = e / 2, e2 = e - e / 2;
                        const float f1 = __int_as_float((127 - e1) << 23), f2 = __int_as_float((127 - e2) << 23);
                        // acc * (sc * 2^-e1) rounds as (acc * sc) * 2^-e1, and the
                        // exact scaling by 2^-e2 fuses with the add: the same bits
                        // as multiplying out and adding, in fewer instructions
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            yacc[q][ps * TP + tt] = fmaf((float)acc[q][tt] * (sc[q] * f1), f2, yacc[q][ps * TP + tt]);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0 && !aborted) mbar_arrive(&s_empty[slot]);
        if (++g == nu) { g = 0; ++t; }
    }
    flush(t_prev);

    // Shared tiles: one ticket each; the CTA that arrives last adds the
    // partial sums of every CTA that owns a unit of the tile (the host sizes
    // the grid so that no CTA's range is empty).
    if (pend0 < 0 && pend1 < 0) return;
    __threadfence();
    named_bar_sync(1, kGemvDecThreads);
    if (tid == 0) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int pt = i ? pend1 : pend0;
            int is_last = 0;
            if (pt >= 0 && !s_misc[3]) {
                const int64_t ut0 = (int64_t)pt * nu;
                const int first = cta_of(ut0, G, C, W, nu, s_offs, kIntUnitBlocks);
                const int last = cta_of(ut0 + nu - 1, G, C, W, nu, s_offs, kIntUnitBlocks);
                is_last = (atomicAdd(&p.tickets[pt], 1) == last - first);
            }
            s_misc[1 + i] = is_last;
        }
    }
    named_bar_sync(1, kGemvDecThreads);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        if (!s_misc[1 + i]) continue;
        __threadfence();
        const int tt = i ? pend1 : pend0;
        const int64_t ut0 = (int64_t)tt * nu;
        const int first = cta_of(ut0, G, C, W, nu, s_offs, kIntUnitBlocks);
        const int last = cta_of(ut0 + nu - 1, G, C, W, nu, s_offs, kIntUnitBlocks);
        const int ncol = p.N - tt * kGemvTileCols;
        const bool first_before = (tt > 0) && cta_of(ut0 - 1, G, C, W, nu, s_offs, kIntUnitBlocks) == first;
        for (int e = tid; e < M * kGemvTileCols; e += kGemvDecThreads) {
            const int tok = e / kGemvTileCols, cl = e - tok * kGemvTileCols;
            if (cl >= ncol) continue;
            float sum = 0.f;
            for (int cc = first; cc <= last; ++cc) {
                const int wc = (cc == first && first_before) ? 1 : 0;
                sum += __ldcg(p.slots + ((size_t)cc * 2 + wc) * (MP * kGemvTileCols) + tok * kGemvTileCols + cl);
            }
            p.y[(size_t)tok * p.N + (size_t)tt * kGemvTileCols + cl] = __float2half_rn(sum);
        }
        if (tid == 0) p.tickets[tt] = 0;
    }
}

}  // namespace qg
