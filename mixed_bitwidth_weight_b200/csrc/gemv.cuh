// Split-K GEMV for decode (M <= 16): y = x[:, perm] . dequant(Wq).
//
// The pages describe decode as bound by memory bandwidth: tokens are generated
// "as fast as memory bandwidth allows" by a kernel "near the memory-bandwidth
// limit" (navi2ai ExLlamaV3 page, "项目概述" and "核心能力").  This kernel
// streams the packed words at HBM speed on B200.  Two kernels per call:
//
// 1. xprep_kernel gathers the activations once through perm, in the order the
//    decoder emits codes (code_of_k), pre-scaled by 2^-P, laid out as the
//    tensor core's B operand.
// 2. gemv_kernel, launched as a programmatic dependent of xprep_kernel: it
//    starts setting up at once and waits for xprep only before it copies data.
//
// Decode without a conversion step.  A code q at mantissa bits [P, P+b) of a
// 16-bit half ORed with 0x6400 is the fp16 number h = 1024 + q * 2^P (one
// lop3 or prmt per two codes); one fp16x2 subtraction of 1024 + z 2^P, exact,
// leaves (q - z) 2^P.  With x' = x * 2^-P as the other operand every product
// is x (q - z) exactly, so the group sum needs no correction term: an
// activation outlier over a weight row at its zero point adds exactly zero,
// and nothing large is subtracted after the accumulation.
//
// Tensor cores.  Each decoder thread owns one output column (one TMEM lane)
// and writes the decoded codes of its column straight into tensor memory with
// tcgen05.st; one thread issues tcgen05.mma (kind::f16, M = 128 columns,
// N = 16 tokens, K = 16) with A read from TMEM and B = the staged activations
// in shared memory, accumulating one 128-row group in fp32 in TMEM.  The
// decoder threads then read their column's group sum back (tcgen05.ld),
// and apply the (group, column) scale.  The legacy
// warp-level mma.sync path is not used: on sm_100 it costs about a dozen
// instructions per MMA, which made decode issue-bound.
//
// Work split.  W is cut into 256-column tiles; a unit is (tile, 128-row group)
// and costs the group's packed word rows plus its scale row.  Units are ordered
// tile-major and cut into gridDim.x contiguous ranges of equal cost, so every
// SM streams the same number of bytes whatever the width mix.  The grid is
// capped so that every range holds at least one unit.  A tile covered by
// several CTAs is finished by the last of them to arrive (an atomic ticket, no
// waiting): partial sums go to workspace slots and that CTA adds them in CTA
// order, so results are deterministic.
//
// Roles.  Warps 0-7: decoders and epilogue, thread t = column t of the tile
// (TMEM lane t % 128 of subtile t / 128).  Warp 8: producer, one lane copies
// each unit's scale row, word rows and activation records with
// cp.async.bulk into a ring of shared-memory rows.  Warp 9: TMEM allocation
// and, on one lane, the MMA issue.
#pragma once

#include "pack_dequant.cuh"

namespace qg {

constexpr int kGemvTileCols = 256;
constexpr int kGemvDecWarps = 8;
constexpr int kGemvDecThreads = kGemvDecWarps * 32;
constexpr int kGemvProducerWarp = 8;
constexpr int kGemvMmaWarp = 9;
constexpr int kGemvThreads = kGemvDecThreads + 64;
constexpr int kGemvRowBytes = (kGemvTileCols + 8) * 4;  // one ring row (1056 B)
constexpr int kGemvSlots = 16;                          // units in flight
constexpr int kGemvMaxRing = 200;                       // ring rows (cap)
constexpr int kGemvMinRing = 80;                        // several units of <= 37 rows
constexpr int kGemvGroupBlocks = kGroupRows / kBlockRows;  // 4
constexpr int kGemvAStages = 3;
constexpr uint32_t kGemvTmemCols = 512;
constexpr int kGemvDCol = kGemvAStages * 128;           // first TMEM column of the D buffers

struct GemvParams {
    const __half* xdec;    // [nb][4][MP][8] activations in decoder order, scaled by 2^-P
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
};

struct XprepParams {
    const void* x;
    const int32_t* perm;
    const uint8_t* bits;
    const int32_t* offs;
    __half* xdec;
    int* xshift;
    int M, K, nb, mp, x_bf16;
};

// Code index (0..31 within a block) that decode_block<b> emits at position k
// (pair k/2, half k%2), and the mantissa bit P at which that code sits.
QG_DEV int code_of_k(int b, int k) {
    const int j = k >> 1, h = k & 1;
    switch (b) {
        case 2: return 16 * (j >> 3) + 4 * ((j & 7) >> 2) + (j & 3) + 8 * h;
        case 4: return 8 * (j >> 2) + (j & 3) + 4 * h;
        case 8: return 4 * (j >> 1) + (j & 1) + 2 * h;
        default: return 8 * (j >> 2) + (j & 3) + 4 * h;  // 3, 5, 6
    }
}

// Mantissa bit P of the codes in fp16x2 value j of a block (both halves).
__host__ __device__ constexpr int shift_of_pair(int b, int j) {
    return b == 2 ? 2 * (j & 3)
         : b == 3 ? (((j & 3) == 1) ? 3 : ((j & 3) == 2) ? 6 : 0)
         : b == 4 ? ((j & 1) ? 4 : 0)
         : b == 5 ? ((j & 1) ? 5 : 0)
         : 0;  // 6, 8
}
QG_DEV int shift_of_k(int b, int k) { return shift_of_pair(b, k >> 1); }

// fp16x2 bits of 1024 + z * 2^P in both halves, z = 2^(b-1): the bias that
// fp16x2 value j of a block carries.
__host__ __device__ constexpr uint32_t bias_of_pair(int b, int j) {
    return (0x6400u | (1u << (b - 1 + shift_of_pair(b, j)))) * 0x10001u;
}

QG_DEV uint32_t hsub2_u32(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// The 32 codes of one block in one column as 16 fp16x2 values
// h = 1024 + q * 2^P, in the order code_of_k describes.  w points at word 0
// of the block in this column; word i is at w + i * kGemvRowBytes.
template <int B>
QG_DEV void decode_block_biased(const uint8_t* w, uint32_t (&P)[16]) {
    auto word = [&](int i) { return *reinterpret_cast<const uint32_t*>(w + i * kGemvRowBytes); };
    if constexpr (B == 2) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const uint32_t v = word(i), v8 = v >> 8;
            P[8 * i + 0] = lop3_mask_magic<0x00030003u>(v);
            P[8 * i + 1] = lop3_mask_magic<0x000C000Cu>(v);
            P[8 * i + 2] = lop3_mask_magic<0x00300030u>(v);
            P[8 * i + 3] = lop3_mask_magic<0x00C000C0u>(v);
            P[8 * i + 4] = lop3_mask_magic<0x00030003u>(v8);
            P[8 * i + 5] = lop3_mask_magic<0x000C000Cu>(v8);
            P[8 * i + 6] = lop3_mask_magic<0x00300030u>(v8);
            P[8 * i + 7] = lop3_mask_magic<0x00C000C0u>(v8);
        }
    } else if constexpr (B == 3) {
        const uint32_t w0 = word(0), w1 = word(1), w2 = word(2);
        const uint32_t X[4] = {w0, __funnelshift_r(w0, w1, 24), __funnelshift_r(w1, w2, 16), w2 >> 8};
#pragma unroll
        for (int c = 0; c < 4; ++c) {  // codes 8c + i at bits 3i of X[c]
            const uint32_t u = (X[c] & 0xFFFFu) | ((X[c] << 4) & 0xFFFF0000u);
            P[4 * c + 0] = lop3_mask_magic<0x00070007u>(u);
            P[4 * c + 1] = lop3_mask_magic<0x00380038u>(u);
            P[4 * c + 2] = lop3_mask_magic<0x01C001C0u>(u);
            P[4 * c + 3] = lop3_mask_magic<0x00070007u>(u >> 9);
        }
    } else if constexpr (B == 4) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t v = word(i), v2 = v >> 8;
            P[4 * i + 0] = lop3_mask_magic<0x000F000Fu>(v);
            P[4 * i + 1] = lop3_mask_magic<0x00F000F0u>(v);
            P[4 * i + 2] = lop3_mask_magic<0x000F000Fu>(v2);
            P[4 * i + 3] = lop3_mask_magic<0x00F000F0u>(v2);
        }
    } else if constexpr (B == 5) {
        uint32_t wd[5];
#pragma unroll
        for (int i = 0; i < 5; ++i) wd[i] = word(i);
#pragma unroll
        for (int c = 0; c < 4; ++c) {  // codes 8c + i at bits 5i of X
            const uint64_t X = ((((uint64_t)wd[c + 1]) << 32) | wd[c]) >> (8 * c);
            const uint32_t u1 = prmt_i<0x5410>((uint32_t)X, (uint32_t)(X >> 20));
            const uint32_t u2 = prmt_i<0x5410>((uint32_t)(X >> 10), (uint32_t)(X >> 30));
            P[4 * c + 0] = lop3_mask_magic<0x001F001Fu>(u1);
            P[4 * c + 1] = lop3_mask_magic<0x03E003E0u>(u1);
            P[4 * c + 2] = lop3_mask_magic<0x001F001Fu>(u2);
            P[4 * c + 3] = lop3_mask_magic<0x03E003E0u>(u2);
        }
    } else if constexpr (B == 6) {
        uint32_t wd[6];
#pragma unroll
        for (int i = 0; i < 6; ++i) wd[i] = word(i);
#pragma unroll
        for (int c = 0; c < 4; ++c) {  // codes 8c + i at bits 6i of X
            const int lo = (c < 2) ? c : c + 1;
            const uint64_t X = ((((uint64_t)wd[lo + 1]) << 32) | wd[lo]) >> ((c & 1) * 16);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                P[4 * c + i] = lop3_mask_magic<0x003F003Fu>(
                    prmt_i<0x5410>((uint32_t)(X >> (6 * i)), (uint32_t)(X >> (6 * i + 24))));
        }
    } else {  // B == 8
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t v = word(i);
            P[2 * i + 0] = prmt_i<0x4240>(v, 0x64646464u);
            P[2 * i + 1] = prmt_i<0x4341>(v, 0x64646464u);
        }
    }
}

// The 32 codes of one block in one column as 16 fp16x2 values
// (q - z) * 2^P, in the order code_of_k describes.  w points at word 0 of the
// block in this column; word i is at w + i * kGemvRowBytes.
template <int B>
QG_DEV void decode_block(const uint8_t* w, uint32_t (&P)[16]) {
    decode_block_biased<B>(w, P);
#pragma unroll
    for (int j = 0; j < 16; ++j) P[j] = hsub2_u32(P[j], bias_of_pair(B, j));  // exact
}

// A full group of 4 blocks of width B: decode each block of this thread's
// column and store it to the TMEM A stage (16 columns per block).  w0 = the
// group's first word row at this column.
template <int B>
QG_DEV void decode_group(const uint8_t* w0, uint32_t ta) {
#pragma unroll
    for (int i = 0; i < kGemvGroupBlocks; ++i) {
        uint32_t P[16];
        decode_block<B>(w0 + i * B * kGemvRowBytes, P);
        tmem_st16(ta + i * 16, P);
    }
}

// Units are numbered t*ng + g (ng units per tile of bpu blocks each; four
// blocks = one 128-row group by default).  A unit's cost is its word rows plus
// one, so the cost prefix of (t, g) is t*(W + ng) + offs[bpu*g] + g, with W
// the word rows of one tile.  CTA i owns the units whose prefix lies in
// [ceil(i*C/G), ceil((i+1)*C/G)), C = tiles * (W + ng).
QG_DEV int64_t unit_start(int64_t i, int64_t G, int64_t C, int64_t W, int nb, int ng, int tiles,
                          const int32_t* s_offs, int bpu = kGemvGroupBlocks) {
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
        if (s_offs[min(mid * bpu, nb)] + mid >= rem) hi = mid; else lo = mid + 1;
    }
    return t * ng + lo;  // lo == ng rolls over to the next tile's group 0
}

// CTA that owns unit u.
QG_DEV int cta_of(int64_t u, int64_t G, int64_t C, int64_t W, int ng, const int32_t* s_offs,
                  int bpu = kGemvGroupBlocks) {
    const int64_t t = u / ng;
    const int g = (int)(u - t * ng);
    const int64_t pos = t * (W + ng) + s_offs[g * bpu] + g;
    if (C * G < (1ll << 32)) return (int)(((uint32_t)pos * (uint32_t)G) / (uint32_t)C);
    return (int)((pos * G) / C);
}

// Ring rows of a unit, contiguous; a unit that would cross the end of the ring
// starts at row 0 instead.  `pos` is the next free row, `total` a monotone
// count of rows used (skipped tails included); producer and consumers replay
// the same sequence.
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

// Ring rows of a unit with `wrows` word rows and `nblk` blocks: the scale row
// (its first 512 bytes hold the scales), the word rows, then the
// activation records (64 * MP bytes per block).
QG_DEV int unit_rows(int wrows, int nblk, int mp) {
    return 1 + wrows + (nblk * 64 * mp + kGemvRowBytes - 1) / kGemvRowBytes;
}

// ------------------------------------------------------------------ xprep
// One warp per block: lane k = position in the decoder's order.  Writes the
// activation of every token (scaled by 2^-P) into the block's record
// [4 k-chunks][MP tokens][8], the B-operand layout of the MMA (tokens >= M
// are zeros).  bf16 input is first scaled per
// row by 2^-shift so that the row's largest magnitude lands in [2^14, 2^15).
__global__ void __launch_bounds__(256) xprep_kernel(const XprepParams p) {
    asm volatile("griddepcontrol.launch_dependents;");
    __shared__ int s_shift[16];
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
    int src = 0, P = 0;
    if (live) {
        P = shift_of_k(b, lane);
        src = p.perm[j * kBlockRows + code_of_k(b, lane)];
        if (src < 0 || src >= p.K) {
            set_dev_error(QGEMM_DEV_BAD_PERM);
            src = 0;
        }
    }
    const float inv2p = __int_as_float((127 - P) << 23);
    __half* rec = p.xdec + (size_t)j * 4 * p.mp * 8;
    for (int m = 0; m < p.mp; ++m) {
        __half xs = __float2half_rn(0.f);
        if (live && m < p.M) {
            const uint16_t raw = reinterpret_cast<const uint16_t*>(p.x)[(size_t)m * p.K + src];
            float v;
            if (p.x_bf16) {
                const int sh = s_shift[m];
                v = __uint_as_float((uint32_t)raw << 16) * __int_as_float((127 - sh / 2) << 23) *
                    __int_as_float((127 - (sh - sh / 2)) << 23);
            } else {
                v = __half2float(__ushort_as_half(raw));
            }
            xs = __float2half_rn(v * inv2p);  // exact unless below fp16 normals
        }
        if (live) rec[((lane >> 3) * p.mp + m) * 8 + (lane & 7)] = xs;
    }
}

// -------------------------------------------------------------------- GEMV
template <int MT>
__global__ void __launch_bounds__(kGemvThreads, 1) gemv_kernel(const GemvParams p) {
    constexpr int MP = MT * 8;
    constexpr int REC = 64 * MP;  // activation record bytes per block
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nb = p.nb, ng = p.ng, M = p.M;

    int32_t* s_offs = reinterpret_cast<int32_t*>(smem);
    size_t o = ((size_t)(nb + 1) * 4 + 15) & ~(size_t)15;
    uint64_t* s_full = reinterpret_cast<uint64_t*>(smem + o);   // ring slot filled
    o += kGemvSlots * 8;
    uint64_t* s_empty = reinterpret_cast<uint64_t*>(smem + o);  // ring slot released
    o += kGemvSlots * 8;
    uint64_t* s_afull = reinterpret_cast<uint64_t*>(smem + o);  // TMEM A stage written
    o += kGemvAStages * 8;
    uint64_t* s_aempty = reinterpret_cast<uint64_t*>(smem + o); // TMEM A stage consumed
    o += kGemvAStages * 8;
    uint64_t* s_dfull = reinterpret_cast<uint64_t*>(smem + o);  // TMEM D buffer ready
    o += 2 * 8;
    uint64_t* s_dempty = reinterpret_cast<uint64_t*>(smem + o); // TMEM D buffer read
    o += 2 * 8;
    uint64_t* s_final = reinterpret_cast<uint64_t*>(smem + o);  // every issued MMA done
    o += 8;
    int* s_misc = reinterpret_cast<int*>(smem + o);  // bad schedule, last flag, abort, tmem base
    int* s_shift = s_misc + 16;
    o += 128;
    o = (o + 127) & ~(size_t)127;
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
            mbar_init(&s_empty[i], kGemvDecWarps + 1);  // decoders + the MMA commit
        }
        for (int i = 0; i < kGemvAStages; ++i) {
            mbar_init(&s_afull[i], kGemvDecWarps);
            mbar_init(&s_aempty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_dfull[i], 1);
            mbar_init(&s_dempty[i], kGemvDecWarps);
        }
        mbar_init(s_final, 1);
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

    // =================================================== producer warp
    if (warp == kGemvProducerWarp) {
        if (lane != 0) return;
        asm volatile("griddepcontrol.wait;" ::: "memory");  // activations come from xprep
        int pos = 0, pos_rel = 0;
        int64_t total = 0, total_rel = 0;
        int k_rel = 0, g_rel = gf;
        bool ok = true;
        int k = 0;
        int t = t0, g = gf;
        for (; k < nunits && ok; ++k) {
            const int j0 = g * kGemvGroupBlocks, j1 = min(j0 + kGemvGroupBlocks, nb);
            const int nblk = j1 - j0;
            const int wrows = s_offs[j1] - s_offs[j0];
            const int need = unit_rows(wrows, nblk, MP);
            int ppos = pos;
            int64_t ptotal = total;
            ring_alloc(ppos, ptotal, need, R);
            while (k - k_rel >= kGemvSlots || ptotal - total_rel > R) {
                if (!mbar_wait(&s_empty[k_rel & (kGemvSlots - 1)], (uint32_t)((k_rel / kGemvSlots) & 1))) {
                    ok = false;
                    break;
                }
                const int jr0 = g_rel * kGemvGroupBlocks, jr1 = min(jr0 + kGemvGroupBlocks, nb);
                ring_alloc(pos_rel, total_rel, unit_rows(s_offs[jr1] - s_offs[jr0], jr1 - jr0, MP), R);
                ++k_rel;
                if (++g_rel == ng) g_rel = 0;
            }
            if (!ok) break;
            const int row = ring_alloc(pos, total, need, R);
            const int slot = k & (kGemvSlots - 1);
            const int cols = min(kGemvTileCols, p.N - t * kGemvTileCols);
            mbar_arrive_expect_tx(&s_full[slot], (uint32_t)(cols * 2 + wrows * cols * 4 + nblk * REC));
            uint8_t* dst = s_ring + (size_t)row * kGemvRowBytes;
            bulk_g2s(dst, p.scales + (size_t)g * p.N + (size_t)t * kGemvTileCols, (uint32_t)cols * 2,
                     &s_full[slot]);
            const uint32_t* src = p.qw + (size_t)s_offs[j0] * p.N + (size_t)t * kGemvTileCols;
            for (int r = 0; r < wrows; ++r)
                bulk_g2s(dst + (size_t)(r + 1) * kGemvRowBytes, src + (size_t)r * p.N, (uint32_t)cols * 4,
                         &s_full[slot]);
            bulk_g2s(dst + (size_t)(1 + wrows) * kGemvRowBytes, p.xdec + (size_t)j0 * (REC / 2),
                     (uint32_t)nblk * REC, &s_full[slot]);
            if (++g == ng) { g = 0; ++t; }
        }
        if (!ok) {
            s_misc[2] = 1;
            // let copies already in flight land before the CTA can exit
            for (int kk = k_rel; kk < k; ++kk)
                mbar_wait(&s_full[kk & (kGemvSlots - 1)], (uint32_t)((kk / kGemvSlots) & 1));
        }
        return;
    }

    // ---- TMEM allocation (warp 9), handed to everyone through shared memory
    if (warp == kGemvMmaWarp) {
        tmem_alloc(reinterpret_cast<uint32_t*>(&s_misc[3]), kGemvTmemCols);
        tmem_relinquish();
        tc_fence_before();
    }
    named_bar_sync(2, kGemvDecThreads + 32);
    tc_fence_after();
    const uint32_t tmem = (uint32_t)s_misc[3];

    // =================================================== MMA issue (warp 9)
    if (warp == kGemvMmaWarp) {
        if (lane == 0) {
            constexpr uint32_t kIdesc = idesc_f16(128, 16);
            const uint32_t lbo = MP * 16, sbo = (MP == 16) ? 128 : 0;  // 8-token groups alias for M <= 8
            int pos = 0;
            int64_t total = 0;
            int g = gf;
            for (int k = 0; k < nunits; ++k) {
                const int j0 = g * kGemvGroupBlocks, j1 = min(j0 + kGemvGroupBlocks, nb);
                const int nblk = j1 - j0;
                const int wrows = s_offs[j1] - s_offs[j0];
                const int row = ring_alloc(pos, total, unit_rows(wrows, nblk, MP), R);
                const int s = k % kGemvAStages, buf = k & 1;
                bool ok = !s_misc[2] && mbar_wait(&s_afull[s], (uint32_t)((k / kGemvAStages) & 1));
                if (ok && k >= 2) ok = mbar_wait(&s_dempty[buf], (uint32_t)(((k >> 1) - 1) & 1));
                if (!ok) {
                    s_misc[2] = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t xrec = smem_u32(s_ring + (size_t)(row + 1 + wrows) * kGemvRowBytes);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t d = tmem + kGemvDCol + buf * 32 + h * 16;
                    const uint32_t a = tmem + s * 128 + h * 64;
                    for (int i = 0; i < nblk; ++i)
#pragma unroll
                        for (int kh = 0; kh < 2; ++kh)
                            tc_mma_ts(d, a + i * 16 + kh * 8,
                                      smem_desc(xrec + i * REC + kh * 2 * lbo, lbo, sbo, 0), kIdesc,
                                      (i | kh) != 0);
                }
                tc_commit(&s_aempty[s]);
                tc_commit(&s_dfull[buf]);
                tc_commit(&s_empty[k & (kGemvSlots - 1)]);
                if (++g == ng) g = 0;
            }
            // every issued MMA completes before the CTA may free TMEM
            tc_commit(s_final);
            mbar_wait(s_final, 0);
        }
        __syncwarp();
        named_bar_sync(3, kGemvDecThreads + 32);
        tc_fence_after();
        tmem_dealloc(tmem, kGemvTmemCols);
        return;
    }

    // =================================================== decoder warps 0-7
    const int ctid = tid;                       // column of the tile
    const uint32_t tlane = (uint32_t)(32 * (warp & 3)) << 16;
    const int sub = warp >> 2;                  // 128-column subtile
    float acc[MP];
#pragma unroll
    for (int i = 0; i < MP; ++i) acc[i] = 0.f;
    bool aborted = false;

    auto out_scale = [&](float v, int tok) -> float {
        const int sh = s_shift[tok];
        if (sh == 0) return v;
        return v * __int_as_float((127 + sh / 2) << 23) * __int_as_float((127 + (sh - sh / 2)) << 23);
    };

    auto flush = [&](int tt) {
        const int64_t ut0 = (int64_t)tt * ng;
        const int first = cta_of(ut0, G, C, W, ng, s_offs);
        const int last = cta_of(ut0 + ng - 1, G, C, W, ng, s_offs);
        const int ncol = p.N - tt * kGemvTileCols;
        if (first == last) {
            if (ctid < ncol && !aborted) {
#pragma unroll
                for (int tok = 0; tok < MP; ++tok)
                    if (tok < M)
                        p.y[(size_t)tok * p.N + (size_t)tt * kGemvTileCols + ctid] =
                            __float2half_rn(out_scale(acc[tok], tok));
            }
            return;
        }
        const int which = (u0 < ut0) ? 1 : 0;
        float* my = p.slots + ((size_t)blockIdx.x * 2 + which) * (MP * kGemvTileCols);
#pragma unroll
        for (int tok = 0; tok < MP; ++tok)
            if (tok < M) my[tok * kGemvTileCols + ctid] = out_scale(acc[tok], tok);
        __threadfence();
        named_bar_sync(1, kGemvDecThreads);
        if (ctid == 0) {
            // every CTA in [first, last] owns a unit of this tile: the host sizes
            // the grid so that no CTA's range is empty
            int is_last = 0;
            if (!s_misc[2]) is_last = (atomicAdd(&p.tickets[tt], 1) == last - first);
            s_misc[1] = is_last;
        }
        named_bar_sync(1, kGemvDecThreads);
        if (s_misc[1]) {
            __threadfence();
            const bool first_before = (tt > 0) && cta_of(ut0 - 1, G, C, W, ng, s_offs) == first;
            if (ctid < ncol)
                for (int tok = 0; tok < M; ++tok) {
                    float s = 0.f;
                    for (int cc = first; cc <= last; ++cc) {
                        const int wc = (cc == first && first_before) ? 1 : 0;
                        s += __ldcg(p.slots + ((size_t)cc * 2 + wc) * (MP * kGemvTileCols) +
                                    tok * kGemvTileCols + ctid);
                    }
                    p.y[(size_t)tok * p.N + (size_t)tt * kGemvTileCols + ctid] = __float2half_rn(s);
                }
            if (ctid == 0) p.tickets[tt] = 0;
        }
        named_bar_sync(1, kGemvDecThreads);
    };

    // epilogue of unit k: group sum from TMEM times the scale
    float prev_sc = 0.f;
    auto epilogue = [&](int k) {
        const int buf = k & 1;
        if (!aborted && !s_misc[2] && mbar_wait(&s_dfull[buf], (uint32_t)((k >> 1) & 1))) {
            tc_fence_after();
            float d[MP];
            if constexpr (MP == 16) tmem_ld16(tmem + tlane + kGemvDCol + buf * 32 + sub * 16, d);
            else tmem_ld8(tmem + tlane + kGemvDCol + buf * 32 + sub * 16, d);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_dempty[buf]);
#pragma unroll
            for (int tok = 0; tok < MP; ++tok) acc[tok] = fmaf(prev_sc, d[tok], acc[tok]);
        } else {
            aborted = true;
            s_misc[2] = 1;
        }
    };

    int pos = 0;
    int64_t total = 0;
    int t = t0, g = gf, t_prev = t0;
    bool have_shift = false;
    for (int k = 0; k < nunits; ++k) {
        const int j0 = g * kGemvGroupBlocks, j1 = min(j0 + kGemvGroupBlocks, nb);
        const int nblk = j1 - j0;
        const int o0 = s_offs[j0];
        const int row = ring_alloc(pos, total, unit_rows(s_offs[j1] - o0, nblk, MP), R);
        const int slot = k & (kGemvSlots - 1);
        const int s = k % kGemvAStages;
        float sc = 0.f;
        if (!aborted && (s_misc[2] || !mbar_wait(&s_full[slot], (uint32_t)((k / kGemvSlots) & 1)))) {
            aborted = true;
            s_misc[2] = 1;
        }
        if (!have_shift) {  // row shifts written by the xprep grid
            asm volatile("griddepcontrol.wait;" ::: "memory");
            if (ctid < 16) s_shift[ctid] = p.xshift[ctid];
            have_shift = true;
        }
        if (!aborted && k >= kGemvAStages &&
            !mbar_wait(&s_aempty[s], (uint32_t)(((k / kGemvAStages) - 1) & 1))) {
            aborted = true;
            s_misc[2] = 1;
        }
        if (!aborted) {
            const uint8_t* ub = s_ring + (size_t)row * kGemvRowBytes;
            sc = __half2float(reinterpret_cast<const __half*>(ub)[ctid]);
            const uint8_t* wcol = ub + kGemvRowBytes + ctid * 4;
            const uint32_t ta = tmem + tlane + s * 128 + sub * 64;
            const int b0 = s_offs[j0 + 1] - o0;
            const bool uniform = (nblk == kGemvGroupBlocks) && (s_offs[j1] - o0 == 4 * b0) &&
                                 (s_offs[j0 + 2] - o0 == 2 * b0) && (s_offs[j0 + 3] - o0 == 3 * b0);
            if (uniform) {  // one straight-line decode + store sequence per width
                switch (b0) {
                    case 2: decode_group<2>(wcol, ta); break;
                    case 3: decode_group<3>(wcol, ta); break;
                    case 4: decode_group<4>(wcol, ta); break;
                    case 5: decode_group<5>(wcol, ta); break;
                    case 6: decode_group<6>(wcol, ta); break;
                    default: decode_group<8>(wcol, ta); break;
                }
            } else {
                for (int j = j0; j < j1; ++j) {
                    const int b = s_offs[j + 1] - s_offs[j];
                    const uint8_t* wb = wcol + (s_offs[j] - o0) * kGemvRowBytes;
                    uint32_t P[16];
                    switch (b) {
                        case 2: decode_block<2>(wb, P); break;
                        case 3: decode_block<3>(wb, P); break;
                        case 4: decode_block<4>(wb, P); break;
                        case 5: decode_block<5>(wb, P); break;
                        case 6: decode_block<6>(wb, P); break;
                        default: decode_block<8>(wb, P); break;
                    }
                    __syncwarp();
                    tmem_st16(ta + (j - j0) * 16, P);
                }
            }
            tc_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&s_afull[s]);
                mbar_arrive(&s_empty[slot]);
            }
        }
        if (k > 0) {
            epilogue(k - 1);
            if (t != t_prev) {  // unit k starts a new tile: the previous one is complete
                named_bar_sync(1, kGemvDecThreads);  // s_shift is visible to every decoder
                flush(t_prev);
                t_prev = t;
#pragma unroll
                for (int i = 0; i < MP; ++i) acc[i] = 0.f;
            }
        }
        prev_sc = sc;
        if (++g == ng) { g = 0; ++t; }
    }
    epilogue(nunits - 1);
    named_bar_sync(1, kGemvDecThreads);
    flush(t_prev);
    // TMEM is released by warp 9 once every decoder is done with it
    tc_fence_before();
    named_bar_sync(3, kGemvDecThreads + 32);
}

}  // namespace qg
