// Decode GEMV for M <= 4 tokens on the integer tensor-core MMA:
//   y = x[:, perm] . dequant(Wq),  dequant(q) = (q - 2^(b-1)) * s[group][column]
// (the quantised matrix multiply of the EXL2 format: mixed 2/3/4/5/6/8-bit
// 32-row blocks, one fp16 scale per 128-row group and column; nightvoyager.top
// exllamav2 report, "关键设计决策"; promptquorum "EXL2量化是什么").
//
// Decode streams 2.5-4 bits per weight, so at B200's HBM bandwidth every SM
// must consume about 50-90 codes per clock; unpacking and multiplying on the
// CUDA cores costs about one integer instruction per code and the integer
// pipe cannot sustain that.  Here the multiply-accumulate runs on the tensor
// cores instead (tcgen05.mma kind::i8, M = 128 output columns, N = 16,
// K = 32 rows of one block), and the CUDA cores only place codes in bytes:
//
//   A (TMEM, u8):  per output column, the block's 32 codes as bytes q * 2^P,
//                  one to four logic operations per four codes
//                  (decode_i8.cuh);
//   B (smem, s8):  per block, 32 rows x 16 columns: for token m and digit d,
//                  column 4m + d holds digit d of x_int * 2^(6 - P), where
//                  x_int is the activation rounded to an integer on a grid
//                  of 2^-e (e per 128-row group part and token, putting the
//                  largest magnitude in [2^22, 2^23)) and the digits are the
//                  balanced base-256 digits (each in [-128, 127]);
//   D (TMEM, s32): per group part and column, four digit sums per token;
//                  sum_d 256^d D_d = 64 * sum_k q_k x_int_k exactly.
//
// The zero point enters once per group part and token as the exact integer
// 64 * sum_k 2^(b_k - 1) x_int_k, subtracted in 64-bit before the one
// conversion to fp32; the result times the fp16 scale and 2^(-e-6) is added to
// a fp32 accumulator.  The activation grid is 2^-23 of the largest magnitude of
// its group part, so an outlier activation costs its group mates nothing
// measurable, whatever the weights under it.
//
// Work split: K is cut into S slices of equal word-row count (each slice's
// activation tiles fit in shared memory); each slice has `cps` CTAs (one per
// SM).  A unit is (256-column tile, pair of group parts of the slice): one
// scale-row copy and at most three word-row copies (a tensor copy costs the
// issuing thread about a hundred cycles whatever its size, so units are made
// large).  The units of a slice are cut into one contiguous range per CTA of
// equal cost (word rows + a fixed cost per unit).  Each CTA:
//   - builds the B tiles of its slice from x and perm (16 decoder warps),
//     while warp 16 already streams each unit's scale and word rows into a
//     shared-memory ring with 2D tensor copies;
//   - four decoder sets of four warps (one TMEM lane quarter each) share each
//     unit: set s takes column half s % 2 and group part s / 2.  A set places
//     its part's codes in TMEM (two A stages per set), reads back the previous
//     unit's D (two D buffers per set) into fp32 per-column accumulators, then
//     signals the MMA warps;
//   - two MMA warps (one issuing thread each, sets {0, 2} and {1, 3}) issue
//     one MMA per block;
//   - when the sets leave a tile, their sums meet in shared memory; a tile
//     that other CTAs share goes to the workspace, and the CTA whose ticket
//     completes the tile adds all contributions in a fixed order and writes y
//     (the same bits on every call).
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "decode_i8.cuh"

namespace qg {

constexpr int kI8Half = 128;                   // output columns per MMA (M)
constexpr int kI8TileCols = 256;               // output columns per tile: two halves
constexpr int kI8Sets = 4;                     // decoder sets of four warps
constexpr int kI8DecWarps = 16;
constexpr int kI8DecThreads = kI8DecWarps * 32;
constexpr int kI8MmaWarp = 16;                 // warps 16-19 issue MMAs, one per decoder set
constexpr int kI8ProdWarp = 20;                // copy issuer
constexpr int kI8Threads = 21 * 32;
constexpr int kI8DBufs = 3;                    // D buffers per set (read-back runs two units behind)
constexpr int kI8MaxM = 4;
constexpr int kI8N = 16;                       // MMA N: 4 digits x 4 tokens
constexpr int kI8BTile = 32 * kI8N;            // B bytes per block
constexpr int kI8RowBytes = kI8TileCols * 4;   // ring row: one word row of a tile
constexpr int kI8Slots = 32;                   // units in flight at most
constexpr int kI8BoxMaps = 7;                  // word boxes of 1..64 rows
constexpr int kI8UnitCost = 24;                // fixed cost of a unit, in word rows
constexpr int kI8MaxSlices = 160;
constexpr int kI8MaxParts = 40;                // group parts per slice
constexpr int kI8MaxUnits = (kI8MaxParts + 1) / 2;  // units per tile of a slice
constexpr int kI8MaxBlocks = 128;              // B tiles per CTA (64 KB)
constexpr int kI8ACol = 0;                     // A stage (set, st): cols (2*set+st)*32
constexpr int kI8DCol = 256;                   // D buffer (set, db): 256 + (3*set+db)*16
constexpr int kI8TmemCols = 512;

// Tensor maps: word rows qw[qw_rows][N] uint32 with boxes of 256 columns x
// 2^i rows, and the scales [G][N] fp16 with a box of 256 columns x 2 rows.
struct I8Maps {
    CUtensorMap w[kI8BoxMaps];
    CUtensorMap s;
};

struct I8Params {
    const void* x;
    const int32_t* perm;
    const uint8_t* bits;
    const int32_t* offs;
    int64_t qw_rows;
    __half* y;
    int* tickets;     // [tiles]
    float* partial;   // [grid][maxt][MP][256]
    int M, K, N, nb, tiles;
    int S, cps, maxt;
    int ring_rows, bcap;
    int x_bf16;
};

// Shared-memory carve-up (bytes); the host sizes the launch with the same
// function.
struct I8Smem {
    int offs, bar, misc, rows, exp, slices, parts, pmax, zs, fs, red, b, ring, total;
};

QG_HD I8Smem i8_smem_layout(int nb, int S, int bcap, int ring_rows, int mp, int maxt) {
    I8Smem L;
    int o = 0;
    L.offs = o;
    o += ((nb + 1) * 4 + 15) & ~15;
    L.bar = o;
    o += (2 * kI8Slots + (2 + kI8DBufs + 1) * kI8Sets + 2) * 8;
    L.misc = o;
    o += 64;
    L.rows = o;  // ring row of each unit in flight
    o += kI8Slots * 4;
    L.exp = o;   // contributions each of the CTA's tiles expects
    o += ((maxt * 4) + 15) & ~15;
    L.slices = o;
    o += ((3 * S + 1) * 4 + 15) & ~15;
    L.parts = o;  // part block starts, unit cost prefixes, uniform part widths
    o += ((kI8MaxParts + 1 + kI8MaxUnits + 1 + kI8MaxParts) * 4 + 15) & ~15;
    L.pmax = o;
    o += kI8MaxParts * kI8MaxM * 4;
    L.zs = o;
    o += kI8MaxParts * kI8MaxM * 8;
    L.fs = o;
    o += kI8MaxParts * kI8MaxM * 4;
    L.red = o;
    o += 2 * kI8Sets * mp * kI8Half * 4;
    o = (o + 127) & ~127;
    L.b = o;
    o += bcap * kI8BTile;
    o = (o + 1023) & ~1023;
    L.ring = o;
    o += ring_rows * kI8RowBytes;
    L.total = o;
    return L;
}

// Code -> (slot, bit offset) for every width, packed as slot | P << 8.
struct I8SlotTable {
    uint16_t v[6][32];
};
QG_HD constexpr I8SlotTable i8_make_slot_table() {
    I8SlotTable t{};
    for (int r = 0; r < 32; ++r) {
        t.v[0][r] = (uint16_t)dec_slot_of_code<2>(r);
        t.v[1][r] = (uint16_t)dec_slot_of_code<3>(r);
        t.v[2][r] = (uint16_t)dec_slot_of_code<4>(r);
        t.v[3][r] = (uint16_t)dec_slot_of_code<5>(r);
        t.v[4][r] = (uint16_t)dec_slot_of_code<6>(r);
        t.v[5][r] = (uint16_t)dec_slot_of_code<8>(r);
    }
    return t;
}
__device__ const I8SlotTable kI8Slot = i8_make_slot_table();

// ------------------------------------------------------------ primitives
QG_DEV int i8_ring_alloc(int& pos, int64_t& total, int need, int R) {
    if (pos + need > R) {
        total += R - pos;
        pos = 0;
    }
    const int row = pos;
    pos += need;
    total += need;
    return row;
}

// mbarrier wait (one thread) that gives up when another thread of the CTA has
// aborted, or after about one second (then it records the timeout and aborts
// the CTA).  Between polls the thread sleeps with exponential backoff, so that
// waiting threads leave the shared-memory pipe to the threads doing work.
QG_DEV bool i8_wait(uint64_t* bar, uint32_t parity, volatile int* abort, uint32_t max_ns = 64) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    uint32_t ns = 16;
    for (uint32_t it = 0; it < (1u << 26); ++it) {
        __nanosleep(ns);
        if (mbar_try_wait(bar, parity)) return true;
        if (ns < max_ns) ns <<= 1;
        if ((it & 63) == 63) {
            if (*abort) return false;
            if (globaltimer_ns() - t0 > 1000000000ull) break;
        }
    }
    set_dev_error(QGEMM_DEV_TIMEOUT);
    *abort = 1;
    return false;
}

// Wait without sleeping (one thread): for the MMA issuers, whose reaction time
// is on the critical path of every unit.
QG_DEV bool i8_spin(uint64_t* bar, uint32_t parity, volatile int* abort) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 0; it < (1u << 30); ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 255) == 255) {
            if (*abort) return false;
            if (globaltimer_ns() - t0 > 1000000000ull) break;
        }
    }
    set_dev_error(QGEMM_DEV_TIMEOUT);
    *abort = 1;
    return false;
}

// The same wait for a whole warp: lane 0 polls, the other lanes wait at the
// warp barrier, which also orders what lane 0 acquired before their reads.
QG_DEV bool i8_wait_warp(uint64_t* bar, uint32_t parity, volatile int* abort) {
    bool ok = true;
    if ((threadIdx.x & 31) == 0) ok = i8_wait(bar, parity, abort, 64);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok;
}

QG_DEV void tc_mma_i8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc, bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"((uint32_t)accumulate));
}

// kind::i8 instruction descriptor: D s32 (2 at bit 4), A u8 (0 at bit 7),
// B s8 (1 at bit 10), both K-major, N >> 3 at bit 17, M >> 4 at bit 24.
QG_DEV constexpr uint32_t idesc_i8(int M, int N) {
    return (2u << 4) | (0u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

QG_DEV void tmem_st8u(uint32_t taddr, const uint32_t (&r)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
                 "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]));
}

template <int NC>
QG_DEV void tmem_ld_u(uint32_t taddr, int32_t (&r)[NC]);
template <>
QG_DEV void tmem_ld_u<4>(uint32_t taddr, int32_t (&r)[4]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];\n\t"
                 "tcgen05.wait::ld.sync.aligned;"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr));
}
template <>
QG_DEV void tmem_ld_u<8>(uint32_t taddr, int32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n\t"
                 "tcgen05.wait::ld.sync.aligned;"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
}
template <>
QG_DEV void tmem_ld_u<16>(uint32_t taddr, int32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

// Words of one block (b rows of the ring at this thread's column) -> the
// eight A registers.
QG_DEV void i8_decode(int b, const uint8_t* wp, uint32_t (&r)[8]) {
    uint32_t w[8];
    auto ld = [&](int i) { return *reinterpret_cast<const uint32_t*>(wp + i * kI8RowBytes); };
    switch (b) {
        case 2:
#pragma unroll
            for (int i = 0; i < 2; ++i) w[i] = ld(i);
            decode_block_i8<2>(w, r);
            break;
        case 3:
#pragma unroll
            for (int i = 0; i < 3; ++i) w[i] = ld(i);
            decode_block_i8<3>(w, r);
            break;
        case 4:
#pragma unroll
            for (int i = 0; i < 4; ++i) w[i] = ld(i);
            decode_block_i8<4>(w, r);
            break;
        case 5:
#pragma unroll
            for (int i = 0; i < 5; ++i) w[i] = ld(i);
            decode_block_i8<5>(w, r);
            break;
        case 6:
#pragma unroll
            for (int i = 0; i < 6; ++i) w[i] = ld(i);
            decode_block_i8<6>(w, r);
            break;
        default:
#pragma unroll
            for (int i = 0; i < 8; ++i) r[i] = ld(i);
            break;
    }
}


QG_DEV void tmem_st32u(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
        "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
        "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31]));
}

// A whole group part of four blocks of one width B: all 4B words are loaded
// first (one shared-memory round trip), then placed; the 32 registers are the
// part's A operand.
template <int B>
QG_DEV void i8_decode_part4(const uint8_t* wp, uint32_t (&r)[32]) {
    uint32_t w[4 * B];
#pragma unroll
    for (int i = 0; i < 4 * B; ++i) w[i] = *reinterpret_cast<const uint32_t*>(wp + i * kI8RowBytes);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        uint32_t o[8];
        decode_block_i8<B>(w + k * B, o);
#pragma unroll
        for (int c = 0; c < 8; ++c) r[8 * k + c] = o[c];
    }
}

// Slice bookkeeping: slice sl covers blocks [jb[sl], jb[sl+1]); its units (a
// tile's pairs of group parts) cost ct[sl] per tile in all, and the tile's
// last unit starts at cost lastc[sl].

// First unit of CTA cc (0..cps) of a slice: the first unit whose cost start is
// at least ceil(cc * Ctot / cps).  uc = the slice's unit cost prefixes, Q
// units per tile.
QG_DEV int64_t i8_unit_start(int cc, int cps, int64_t Ct, int64_t T, int Q, const int* uc) {
    const int64_t Ctot = T * Ct;
    const int64_t target = ((int64_t)cc * Ctot + cps - 1) / cps;
    const int64_t t = target / Ct, rem = target - t * Ct;
    if (rem == 0) return t * Q;
    for (int q = 1; q < Q; ++q)
        if (uc[q] >= rem) return t * Q + q;
    return (t + 1) * Q;
}

// Tile of the first unit of CTA cc of a slice (needs only the slice's costs).
QG_DEV int64_t i8_first_tile(int cc, int cps, int64_t Ct, int64_t lastc, int64_t T) {
    const int64_t Ctot = T * Ct;
    const int64_t target = ((int64_t)cc * Ctot + cps - 1) / cps;
    const int64_t t = target / Ct, rem = target - t * Ct;
    return t + (rem > lastc ? 1 : 0);
}

// Block where the last unit of a slice's tile starts.
QG_DEV int i8_last_unit_block(int jb0, int jb1) {
    const int g0 = jb0 >> 2, P = ((jb1 - 1) >> 2) - g0 + 1, p = 2 * ((P + 1) / 2 - 1);
    return p == 0 ? jb0 : 4 * (g0 + p);
}

// ----------------------------------------------------------------- kernel
template <int MP>
__global__ void __launch_bounds__(kI8Threads, 1) gemv_i8_kernel(const I8Params p, const __grid_constant__ I8Maps maps) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nb = p.nb, S = p.S, cps = p.cps, R = p.ring_rows;
    const int64_t T = p.tiles;
    const I8Smem L = i8_smem_layout(nb, S, p.bcap, R, MP, p.maxt);
    int32_t* s_offs = reinterpret_cast<int32_t*>(smem + L.offs);
    uint64_t* s_full = reinterpret_cast<uint64_t*>(smem + L.bar);
    uint64_t* s_empty = s_full + kI8Slots;
    uint64_t* s_afull = s_empty + kI8Slots;       // [set*2 + A stage]
    uint64_t* s_mdone = s_afull + 2 * kI8Sets;    // [set*3 + D buffer]
    uint64_t* s_redfree = s_mdone + kI8DBufs * kI8Sets;  // [2]
    uint64_t* s_fin = s_redfree + 2;              // [4]
    volatile int* s_misc = reinterpret_cast<volatile int*>(smem + L.misc);
    // s_misc: [0] abort, [1] bad schedule, [2..3] set count per red buffer,
    //         [4..7] per-set flags, [8] TMEM base, [9..11] first tile, unit, count
    volatile int* s_row = reinterpret_cast<volatile int*>(smem + L.rows);
    int* s_exp = reinterpret_cast<int*>(smem + L.exp);
    int* s_jb = reinterpret_cast<int*>(smem + L.slices);
    int* s_ct = s_jb + S + 1;
    int* s_lastc = s_ct + S;
    int* s_pj0 = reinterpret_cast<int*>(smem + L.parts);  // own slice: part block starts [P+1]
    int* s_uc = s_pj0 + kI8MaxParts + 1;                   // unit cost prefixes [Q+1]
    int* s_pu = s_uc + kI8MaxUnits + 1;                    // width of a four-block uniform part, else 0 [P]
    int* s_pmax = reinterpret_cast<int*>(smem + L.pmax);   // [part][4]
    long long* s_z = reinterpret_cast<long long*>(smem + L.zs);
    float* s_f = reinterpret_cast<float*>(smem + L.fs);
    float* s_red = reinterpret_cast<float*>(smem + L.red);  // [2][4 sets][MP][128]
    uint8_t* s_b = smem + L.b;
    uint8_t* s_ring = smem + L.ring;

    // the next call may start its prologue during this grid; it waits for
    // this grid's completion before it touches x, y or the workspace
    if (tid == 0) asm volatile("griddepcontrol.launch_dependents;");
    if (warp == kI8ProdWarp && lane == 0) {
#pragma unroll
        for (int i = 0; i < kI8BoxMaps; ++i) asm volatile("prefetch.tensormap [%0];" ::"l"(&maps.w[i]) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&maps.s) : "memory");
    }

    // ---- schedule into shared memory, barriers, TMEM
    if (tid < 8) s_misc[tid] = 0;  // s_misc[8] receives the TMEM address below
    for (int j = tid; j <= nb; j += kI8Threads) s_offs[j] = p.offs[j];
    constexpr int kBitsPerThread = (kMaxK / kBlockRows + kI8Threads - 1) / kI8Threads;
    int my_bits[kBitsPerThread];  // widths of this thread's blocks
#pragma unroll
    for (int r = 0; r < kBitsPerThread; ++r) {
        const int j = tid + r * kI8Threads;
        my_bits[r] = (j < nb) ? (int)p.bits[j] : 0;
    }
    if (warp == kI8MmaWarp) {
        tmem_alloc(reinterpret_cast<uint32_t*>(const_cast<int*>(s_misc + 8)), kI8TmemCols);
        tmem_relinquish();
    }
    if (tid == kI8Threads - 1) {
        for (int i = 0; i < kI8Slots; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&s_empty[i], kI8DecWarps);
        }
        for (int i = 0; i < 2 * kI8Sets; ++i) mbar_init(&s_afull[i], 4);
        for (int i = 0; i < kI8DBufs * kI8Sets; ++i) mbar_init(&s_mdone[i], 1);
        for (int i = 0; i < 2; ++i) mbar_init(&s_redfree[i], 1);
        for (int i = 0; i < kI8Sets; ++i) mbar_init(&s_fin[i], 1);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    {
        // every width must be a format width equal to its offset difference,
        // and the table must end at qw_rows: then every word row the kernel
        // touches is inside qw
        bool bad = false;
#pragma unroll
        for (int r = 0; r < kBitsPerThread; ++r) {
            const int j = tid + r * kI8Threads;
            if (j < nb && (!width_ok(my_bits[r]) || s_offs[j + 1] - s_offs[j] != my_bits[r])) bad = true;
        }
        if (tid == 0 && (s_offs[0] != 0 || (int64_t)s_offs[nb] != p.qw_rows)) bad = true;
        if (bad) atomicOr(const_cast<int*>(&s_misc[1]), 1);
        // slice boundaries: first block whose row offset reaches sl/S of the rows
        const int64_t W = p.qw_rows;
        if (tid <= S) {
            int lo = 0, hi = nb;
            if (tid == 0) hi = 0;
            else if (tid == S) lo = nb;
            else {
                while (lo < hi) {
                    const int mid = (lo + hi) >> 1;
                    if ((int64_t)s_offs[mid] * S >= (int64_t)tid * W) hi = mid;
                    else lo = mid + 1;
                }
            }
            s_jb[tid] = lo;
        }
    }
    __syncthreads();
    const uint32_t tbase = (uint32_t)s_misc[8];
    if (s_misc[1]) {
        if (tid == 0) {
            set_dev_error(QGEMM_DEV_BAD_SCHEDULE);
            asm volatile("griddepcontrol.wait;" ::: "memory");
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (warp == kI8MmaWarp) tmem_dealloc(tbase, kI8TmemCols);
        return;
    }
    if (tid < S) {
        const int jb0 = s_jb[tid], jb1 = s_jb[tid + 1];
        const int P = ((jb1 - 1) >> 2) - (jb0 >> 2) + 1, Q = (P + 1) / 2;
        const int ct = (s_offs[jb1] - s_offs[jb0]) + kI8UnitCost * Q;
        s_ct[tid] = ct;
        s_lastc[tid] = ct - ((s_offs[jb1] - s_offs[i8_last_unit_block(jb0, jb1)]) + kI8UnitCost);
    }
    const int sl = blockIdx.x / cps, cc = blockIdx.x - sl * cps;
    const int jb0 = s_jb[sl], jb1 = s_jb[sl + 1];
    const int P = ((jb1 - 1) >> 2) - (jb0 >> 2) + 1;   // group parts of the slice
    const int Q = (P + 1) / 2;                           // units per tile
    const int nbl = jb1 - jb0;
    if (tid <= P) s_pj0[tid] = (tid == 0) ? jb0 : (tid == P ? jb1 : 4 * ((jb0 >> 2) + tid));
    __syncthreads();
    if (tid <= Q) s_uc[tid] = (s_offs[s_pj0[min(2 * tid, P)]] - s_offs[jb0]) + kI8UnitCost * tid;
    if (tid < P) {
        const int j0 = s_pj0[tid], j1 = s_pj0[tid + 1], b = s_offs[j0 + 1] - s_offs[j0];
        bool uni = (j1 - j0 == 4);
        for (int j = j0 + 1; j < j1; ++j) uni = uni && (s_offs[j + 1] - s_offs[j] == b);
        s_pu[tid] = uni ? b : 0;
    }
    __syncthreads();
    if (tid == 0) {  // the CTA's unit range (64-bit arithmetic, once)
        const int64_t Ct = s_ct[sl];
        const int64_t u0 = i8_unit_start(cc, cps, Ct, T, Q, s_uc);
        const int64_t u1 = i8_unit_start(cc + 1, cps, Ct, T, Q, s_uc);
        s_misc[9] = (int)(u0 / Q);
        s_misc[10] = (int)(u0 - (u0 / Q) * Q);
        s_misc[11] = (int)(u1 - u0);
    }
    __syncthreads();
    const int t_first = s_misc[9], q_first = s_misc[10], nunits = s_misc[11];
    const int ntl = nunits > 0 ? (q_first + nunits - 1) / Q + 1 : 0;  // tiles the CTA touches
    volatile int* abort = s_misc;

    if (warp == kI8ProdWarp) {
        // ======================================= copy issuer (one thread)
        if (lane == 0 && nunits > 0) {
            int pos = 0, pos_rel = 0, k_rel = 0, k = 0;
            int t = t_first, q = q_first, q_rel = q_first;
            int64_t total = 0, total_rel = 0;
            bool ok = true;
            for (; k < nunits && ok; ++k) {
                const int j0 = s_pj0[2 * q], j1 = s_pj0[min(2 * q + 2, P)];
                const int r0 = s_offs[j0], nrows = s_offs[j1] - r0;
                int ppos = pos;
                int64_t ptot = total;
                i8_ring_alloc(ppos, ptot, 1 + nrows, R);
                while (k - k_rel >= kI8Slots || (ptot - total_rel > R && k_rel < k)) {
                    if (!i8_wait(&s_empty[k_rel % kI8Slots], (uint32_t)((k_rel / kI8Slots) & 1), abort)) {
                        ok = false;
                        break;
                    }
                    i8_ring_alloc(pos_rel, total_rel,
                                  1 + s_offs[s_pj0[min(2 * q_rel + 2, P)]] - s_offs[s_pj0[2 * q_rel]], R);
                    if (++q_rel == Q) q_rel = 0;
                    ++k_rel;
                }
                if (!ok) break;
                const int row = i8_ring_alloc(pos, total, 1 + nrows, R);
                s_row[k % kI8Slots] = row;  // published by the arrive below (release)
                uint64_t* bar = &s_full[k % kI8Slots];
                mbar_arrive_expect_tx(bar, (uint32_t)((1 + nrows) * kI8RowBytes));
                uint8_t* dst = s_ring + (size_t)row * kI8RowBytes;
                tma_load_2d(dst, &maps.s, t * kI8TileCols, j0 >> 2, bar);
                int rr = 0;
#pragma unroll
                for (int i = kI8BoxMaps - 1; i >= 0; --i)
                    if (nrows & (1 << i)) {
                        tma_load_2d(dst + (size_t)(1 + rr) * kI8RowBytes, &maps.w[i], t * kI8TileCols, r0 + rr, bar);
                        rr += 1 << i;
                    }
                if (++q == Q) {
                    q = 0;
                    ++t;
                }
            }
            if (!ok) {
                // copies in flight must land before the CTA's shared memory goes away
                for (int kk = k_rel; kk < k; ++kk) {
                    uint64_t* bar = &s_full[kk % kI8Slots];
                    const uint64_t t0 = globaltimer_ns();
                    while (!mbar_try_wait_sleep(bar, (uint32_t)((kk / kI8Slots) & 1), 20000u))
                        if (globaltimer_ns() - t0 > 1000000000ull) break;
                }
            }
        }
    } else if (warp >= kI8MmaWarp) {
        // ======================================= MMA issuers: warp 16 + s serves decoder set s
        named_bar_sync(1, kI8DecThreads + 32 * kI8Sets);  // B tiles ready
        if (lane == 0) {
            const int set = warp - kI8MmaWarp, ph = set >> 1;
            const uint32_t idesc = idesc_i8(kI8Half, kI8N);
            const uint64_t bdesc0 = smem_desc(smem_u32(s_b), 16 * kI8N, 128, 0);
            int q = q_first;
            for (int k = 0; k < nunits; ++k) {
                const int st = k & 1, db = k % kI8DBufs, part = 2 * q + ph;
                if (!i8_spin(&s_afull[2 * set + st], (uint32_t)((k >> 1) & 1), abort)) break;
                tc_fence_after();
                if (part < P) {
                    const int j0 = s_pj0[part], j1 = s_pj0[part + 1];
                    const uint32_t d = tbase + kI8DCol + (uint32_t)((kI8DBufs * set + db) * 16);
                    const uint32_t a = tbase + kI8ACol + (uint32_t)((2 * set + st) * 32);
                    for (int j = j0; j < j1; ++j)
                        tc_mma_i8(d, a + 8 * (j - j0), bdesc0 + (uint64_t)((j - jb0) * (kI8BTile >> 4)), idesc,
                                  j > j0);
                }
                tc_commit(&s_mdone[kI8DBufs * set + db]);
                if (++q == Q) q = 0;
            }
            // every MMA of this thread completes before TMEM is released
            tc_commit(&s_fin[set]);
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait_sleep(&s_fin[set], 0u, 20000u))
                if (globaltimer_ns() - t0 > 1000000000ull) break;
        }
        __syncwarp();
    } else {
        // ======================================= decoder warps 0-15
        const int set = warp >> 2, quarter = warp & 3, col = 32 * quarter + lane;
        const int half = set & 1, ph = set >> 1;     // column half and part of each unit
        const uint32_t tlane = (uint32_t)(32 * quarter) << 16;
        // contributions each touched tile expects (64-bit arithmetic, once per tile)
        if (tid < ntl) {
            const int tt = t_first + tid;
            const int first = (int)((int64_t)tt * cps / T);
            int expected = 0;
            for (int s2 = 0; s2 < S; ++s2) {
                const int64_t c2 = s_ct[s2];
                expected += (int)(((int64_t)tt * c2 + s_lastc[s2]) * cps / (T * c2)) - first + 1;
            }
            s_exp[tid] = expected;
        }
        asm volatile("griddepcontrol.wait;" ::: "memory");  // x may come from the previous grid

        // ---- activation tiles of the slice (B operand), zero points, scales
        {
            uint4* bz = reinterpret_cast<uint4*>(s_b);
            for (int i = tid; i < nbl * (kI8BTile / 16); i += kI8DecThreads) bz[i] = make_uint4(0, 0, 0, 0);
            if (tid < kI8MaxParts * kI8MaxM) {
                s_pmax[tid] = 0;
                s_z[tid] = 0;
            }
        }
        // gathers first (all rounds), then the arithmetic: two memory round trips
        int src[8];
#pragma unroll
        for (int rd = 0; rd < 8; ++rd) {
            const int jl = rd * kI8DecWarps + warp;
            src[rd] = (jl < nbl) ? p.perm[(jb0 + jl) * kBlockRows + lane] : 0;
        }
        float xv[8][MP];
        const uint16_t* xh = static_cast<const uint16_t*>(p.x);
#pragma unroll
        for (int rd = 0; rd < 8; ++rd) {
            const int jl = rd * kI8DecWarps + warp;
            if (src[rd] < 0 || src[rd] >= p.K) {
                set_dev_error(QGEMM_DEV_BAD_PERM);
                src[rd] = 0;
            }
#pragma unroll
            for (int m = 0; m < MP; ++m) {
                xv[rd][m] = 0.f;
                if (jl < nbl && m < p.M) {
                    const uint16_t raw = xh[(size_t)m * p.K + src[rd]];
                    xv[rd][m] = p.x_bf16 ? __uint_as_float((uint32_t)raw << 16) : __half2float(__ushort_as_half(raw));
                }
            }
        }
        named_bar_sync(2, kI8DecThreads);  // B zeroed, part maxima cleared
#pragma unroll
        for (int rd = 0; rd < 8; ++rd) {
            const int jl = rd * kI8DecWarps + warp;
            if (jl >= nbl) continue;
            const int part = ((jb0 + jl) >> 2) - (jb0 >> 2);
#pragma unroll
            for (int m = 0; m < MP; ++m) {
                int a = __float_as_int(fabsf(xv[rd][m]));
                if (a >= 0x7F800000) a = 0x7F7FFFFF;  // inf / nan: the largest finite magnitude
#pragma unroll
                for (int o = 16; o; o >>= 1) a = max(a, __shfl_xor_sync(0xffffffffu, a, o));
                if (lane == 0) atomicMax(&s_pmax[part * kI8MaxM + m], a);
            }
        }
        named_bar_sync(2, kI8DecThreads);
#pragma unroll
        for (int rd = 0; rd < 8; ++rd) {
            const int jl = rd * kI8DecWarps + warp;
            if (jl >= nbl) continue;
            const int j = jb0 + jl;
            const int b = s_offs[j + 1] - s_offs[j];
            const int part = (j >> 2) - (jb0 >> 2);
            const uint32_t so = __ldg(&kI8Slot.v[width_index(b)][lane]);
            const int slot = so & 0xFF, sh = so >> 8;
            uint8_t* bt = s_b + jl * kI8BTile + (slot >> 4) * 256 + (slot & 15);
#pragma unroll
            for (int m = 0; m < MP; ++m) {
                const int E = (s_pmax[part * kI8MaxM + m] >> 23) & 0xFF;
                int xi = 0;
                if (E >= 30) {  // parts whose largest magnitude is below 2^-97 count as zero
                    const int e = 149 - min(E, 254), e1 = e / 2, e2 = e - e1;
                    xi = __float2int_rn(xv[rd][m] * __int_as_float((127 + e1) << 23) * __int_as_float((127 + e2) << 23));
                }
                int v = xi * (1 << (6 - sh));
                const int d0 = (int)(int8_t)(v & 0xFF);
                v = (v - d0) >> 8;
                const int d1 = (int)(int8_t)(v & 0xFF);
                v = (v - d1) >> 8;
                const int d2 = (int)(int8_t)(v & 0xFF);
                const int d3 = (v - d2) >> 8;
                bt[(4 * m + 0) * 16] = (uint8_t)d0;
                bt[(4 * m + 1) * 16] = (uint8_t)d1;
                bt[(4 * m + 2) * 16] = (uint8_t)d2;
                bt[(4 * m + 3) * 16] = (uint8_t)d3;
                int sum = xi;
#pragma unroll
                for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
                if (lane == 0 && sum != 0)
                    atomicAdd(reinterpret_cast<unsigned long long*>(&s_z[part * kI8MaxM + m]),
                              (unsigned long long)((long long)sum * (64ll << (b - 1))));
            }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // B is read by the tensor cores
        named_bar_sync(2, kI8DecThreads);
        if (tid < P * MP) {
            const int part = tid / MP, m = tid - part * MP;
            const int E = (s_pmax[part * kI8MaxM + m] >> 23) & 0xFF;
            s_f[part * kI8MaxM + m] = (E >= 30) ? __int_as_float((min(E, 254) - 28) << 23) : 0.f;  // 2^(E-155)
        }
        named_bar_sync(1, kI8DecThreads + 32 * kI8Sets);  // B tiles ready for the MMA warps
        named_bar_sync(2, kI8DecThreads);       // s_f, s_exp visible to every decoder

        // ---- main loop
        float yacc[MP];
#pragma unroll
        for (int m = 0; m < MP; ++m) yacc[m] = 0.f;
        int cur = t_first;  // tile the accumulators belong to
        bool dead = false;  // this thread stopped working (abort); barriers still run

        // The four sets' sums of tile tt meet in shared memory; the last set
        // to arrive adds them (sets 0 + 2: columns 0-127, sets 1 + 3: columns
        // 128-255) and hands the tile on: y, or the workspace and the tile's
        // ticket.
        auto flush = [&](int tt) {
            const int l = tt - t_first, buf = l & 1;
            if (l >= 2 && !dead && !i8_wait_warp(&s_redfree[buf], (uint32_t)(((l >> 1) - 1) & 1), abort)) dead = true;
            float* rb = s_red + (size_t)buf * kI8Sets * MP * kI8Half;
#pragma unroll
            for (int m = 0; m < MP; ++m) rb[(set * MP + m) * kI8Half + col] = yacc[m];
            named_bar_sync(3 + set, 128);
            if (col == 0) {
                __threadfence_block();
                const int old = atomicAdd(const_cast<int*>(&s_misc[2 + buf]), 1);
                s_misc[4 + set] = (old == kI8Sets - 1);
            }
            named_bar_sync(3 + set, 128);
            if (!s_misc[4 + set]) return;
            // this set reduces tile tt
            __threadfence_block();
            float v[2][MP];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                for (int m = 0; m < MP; ++m)
                    v[hh][m] = rb[(hh * MP + m) * kI8Half + col] + rb[((hh + 2) * MP + m) * kI8Half + col];
            named_bar_sync(3 + set, 128);
            if (col == 0) {
                s_misc[2 + buf] = 0;
                mbar_arrive(&s_redfree[buf]);
            }
            const bool live = !*abort;
            const int expected = s_exp[l];
            const int n0 = tt * kI8TileCols + col;
            if (expected == 1) {
                if (live)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                        for (int m = 0; m < MP; ++m)
                            if (m < p.M && n0 + kI8Half * hh < p.N)
                                p.y[(size_t)m * p.N + n0 + kI8Half * hh] = __float2half_rn(v[hh][m]);
                return;
            }
            float* mine = p.partial + ((size_t)blockIdx.x * p.maxt + l) * MP * kI8TileCols;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                for (int m = 0; m < MP; ++m) mine[m * kI8TileCols + kI8Half * hh + col] = v[hh][m];
            __threadfence();
            named_bar_sync(3 + set, 128);
            if (col == 0) {
                int last = 0;
                if (live) last = (atomicAdd(&p.tickets[tt], 1) == expected - 1);
                s_misc[4 + set] = last;
            }
            named_bar_sync(3 + set, 128);
            if (!s_misc[4 + set]) return;
            __threadfence();
            float sum[2][MP];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                for (int m = 0; m < MP; ++m) sum[hh][m] = 0.f;
            const int first = (int)((int64_t)tt * cps / T);
            for (int s2 = 0; s2 < S; ++s2) {
                const int64_t c2 = s_ct[s2];
                const int last2 = (int)(((int64_t)tt * c2 + s_lastc[s2]) * cps / (T * c2));
                for (int q2 = first; q2 <= last2; ++q2) {
                    const int l2 = tt - (int)i8_first_tile(q2, cps, c2, s_lastc[s2], T);
                    const float* src2 = p.partial + ((size_t)(s2 * cps + q2) * p.maxt + l2) * MP * kI8TileCols;
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                        for (int m = 0; m < MP; ++m) sum[hh][m] += __ldcg(src2 + m * kI8TileCols + kI8Half * hh + col);
                }
            }
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                for (int m = 0; m < MP; ++m)
                    if (m < p.M && n0 + kI8Half * hh < p.N)
                        p.y[(size_t)m * p.N + n0 + kI8Half * hh] = __float2half_rn(sum[hh][m]);
            if (col == 0) p.tickets[tt] = 0;
        };
        auto advance_to = [&](int tt) {
            while (cur < tt) {
                flush(cur);
#pragma unroll
                for (int m = 0; m < MP; ++m) yacc[m] = 0.f;
                ++cur;
            }
        };

        // read back a part's D: digits -> exact 64-bit sum -> fp32, into yacc
        auto readback = [&](int k, int part, int tt, float sc) {
            const int db = k % kI8DBufs;
            if (!dead && !i8_wait_warp(&s_mdone[kI8DBufs * set + db], (uint32_t)((k / kI8DBufs) & 1), abort)) dead = true;
            dead = __any_sync(0xffffffffu, dead);  // tcgen05.ld is warp-collective
            tc_fence_after();
            int32_t dv[4 * MP];
            const bool use = !dead && part < P;
            if (use) tmem_ld_u<4 * MP>(tbase + tlane + kI8DCol + (uint32_t)((kI8DBufs * set + db) * 16), dv);
            tc_fence_before();
            advance_to(tt);
            if (!use) return;
#pragma unroll
            for (int m = 0; m < MP; ++m) {
                const int lo = dv[4 * m] + dv[4 * m + 1] * 256;
                const int hi = dv[4 * m + 2] + dv[4 * m + 3] * 256;
                const long long s64 = (long long)hi * 65536ll + (long long)lo - s_z[part * kI8MaxM + m];
                yacc[m] = fmaf((float)s64, sc * s_f[part * kI8MaxM + m], yacc[m]);
            }
        };

        // Unit k: read back unit k - 2 (its MMAs have had two units' time to
        // finish; it also frees the A stage unit k reuses), then place unit
        // k's codes and hand them to the set's MMA warp.
        int hpart0 = 0, hpart1 = 0, ht0 = 0, ht1 = 0;  // units k - 2 and k - 1 (by parity)
        float hsc0 = 0.f, hsc1 = 0.f;
        int t = t_first, q = q_first;
        for (int k = 0; k < nunits; ++k) {
            const int st = k & 1;
            const int part = 2 * q + ph;
            if (k >= 2) readback(k - 2, st ? hpart1 : hpart0, st ? ht1 : ht0, st ? hsc1 : hsc0);
            float sc = 0.f;
            if (!dead && !i8_wait_warp(&s_full[k % kI8Slots], (uint32_t)((k / kI8Slots) & 1), abort)) dead = true;
            dead = __any_sync(0xffffffffu, dead);  // tcgen05.st is warp-collective
            if (!dead && part < P) {
                const int j0 = s_pj0[part], j1 = s_pj0[part + 1];
                const uint8_t* ub = s_ring + (size_t)s_row[k % kI8Slots] * kI8RowBytes;
                sc = __half2float(reinterpret_cast<const __half*>(ub)[ph * kI8TileCols + half * kI8Half + col]);
                const int o0 = s_offs[j0];
                const uint8_t* wp = ub + (size_t)(1 + o0 - s_offs[s_pj0[2 * q]]) * kI8RowBytes + (half * kI8Half + col) * 4;
                const uint32_t ta = tbase + tlane + kI8ACol + (uint32_t)((2 * set + st) * 32);
                const int b = s_pu[part];
                if (b) {  // four blocks of one width
                    uint32_t r[32];
                    switch (b) {
                        case 2: i8_decode_part4<2>(wp, r); break;
                        case 3: i8_decode_part4<3>(wp, r); break;
                        case 4: i8_decode_part4<4>(wp, r); break;
                        case 5: i8_decode_part4<5>(wp, r); break;
                        case 6: i8_decode_part4<6>(wp, r); break;
                        default: i8_decode_part4<8>(wp, r); break;
                    }
                    tmem_st32u(ta, r);
                } else {
                    for (int jj = j0; jj < j1; ++jj) {
                        uint32_t r[8];
                        i8_decode(s_offs[jj + 1] - s_offs[jj], wp + (size_t)(s_offs[jj] - o0) * kI8RowBytes, r);
                        tmem_st8u(ta + 8 * (jj - j0), r);
                    }
                }
            }
            __syncwarp();
            if (lane == 0 && !dead) mbar_arrive(&s_empty[k % kI8Slots]);  // words and scale read
            if (!dead) tc_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0 && !dead) mbar_arrive(&s_afull[2 * set + st]);
            if (st) {
                hpart1 = part;
                ht1 = t;
                hsc1 = sc;
            } else {
                hpart0 = part;
                ht0 = t;
                hsc0 = sc;
            }
            if (++q == Q) {
                q = 0;
                ++t;
            }
        }
        for (int k = max(0, nunits - 2); k < nunits; ++k)
            readback(k, (k & 1) ? hpart1 : hpart0, (k & 1) ? ht1 : ht0, (k & 1) ? hsc1 : hsc0);
        if (ntl > 0) advance_to(t_first + ntl);
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kI8MmaWarp) tmem_dealloc(tbase, kI8TmemCols);
}

}  // namespace qg
