// Pack (codes -> packed words) and dequant (packed words -> fp16 W) kernels.
//
// Format: the EXL2-style mixed-width layout described in include/qgemm.h
// (nightvoyager.top exllamav2 report, "核心价值提炼"; promptquorum
// "EXL2量化是什么").  Both kernels are HBM-bound streaming passes; they are
// not on the decode hot path but make the format usable from the library.
#pragma once

#include "common.cuh"

namespace qg {


// Local consistency of block j of the schedule.  Checking this for every
// block a kernel touches keeps all of its word-row accesses inside
// [0, qw_rows); a kernel that finds a bad block records the error and skips it.
QG_DEV bool block_schedule_ok(const uint8_t* bits, const int32_t* offs, int j, int nb,
                              int64_t qw_rows, int* b_out, int* off_out) {
    const int b = bits[j];
    const int o0 = offs[j], o1 = offs[j + 1];
    bool ok = width_ok(b) && o0 >= 0 && o1 == o0 + b && (int64_t)o1 <= qw_rows;
    if (j == 0) ok = ok && o0 == 0;
    if (j == nb - 1) ok = ok && (int64_t)o1 == qw_rows;
    *b_out = b;
    *off_out = o0;
    return ok;
}

// ------------------------------------------------------------------ pack
// One thread per (block, 4 consecutive columns): reads the block's 32 rows of
// its 4 codes as one 32-bit word each (128 bytes per warp per row) and emits
// the 4 columns' little-endian streams, one 16-byte store per word row.
// N is a multiple of 8, so a thread's 4 columns are all in range.
__global__ void __launch_bounds__(128) pack_kernel(const uint8_t* __restrict__ codes,
                                                   const uint8_t* __restrict__ bits,
                                                   const int32_t* __restrict__ offs, int K,
                                                   int N, int64_t qw_rows,
                                                   uint32_t* __restrict__ qw) {
    const int n0 = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
    const int j = blockIdx.y;
    const int nb = K / kBlockRows;
    if (n0 >= N) return;
    int b, off;
    if (!block_schedule_ok(bits, offs, j, nb, qw_rows, &b, &off)) {
        set_dev_error(QGEMM_DEV_BAD_SCHEDULE);
        return;
    }
    const uint32_t mask = (1u << b) - 1u;
    const uint8_t* src = codes + (size_t)j * kBlockRows * N + n0;
    uint32_t* dst = qw + (size_t)off * N + n0;
    uint32_t rows[kBlockRows];
#pragma unroll
    for (int r = 0; r < kBlockRows; ++r) rows[r] = *reinterpret_cast<const uint32_t*>(src + (size_t)r * N);
    uint64_t acc[4] = {0, 0, 0, 0};
    int nacc = 0, w = 0;
#pragma unroll
    for (int r = 0; r < kBlockRows; ++r) {
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[c] |= (uint64_t)((rows[r] >> (8 * c)) & mask) << nacc;
        nacc += b;
        if (nacc >= 32) {
            *reinterpret_cast<uint4*>(dst + (size_t)w * N) =
                make_uint4((uint32_t)acc[0], (uint32_t)acc[1], (uint32_t)acc[2], (uint32_t)acc[3]);
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[c] >>= 32;
            nacc -= 32;
            ++w;
        }
    }
}

// ---------------------------------------------------------------- dequant
// One thread per (block, 4 consecutive columns).  Each code is decoded from a
// 64-bit window of two stream words; the weight (q - 2^(b-1)) * s is exact in
// fp32 (at most 19 significant bits, also for subnormal fp16 scales), so the
// single cvt.rn to fp16 gives the correctly rounded result.
template <int B>
QG_DEV void dequant_block4(const uint32_t* __restrict__ src, const __half* __restrict__ srow,
                           __half* __restrict__ dst, int N) {
    uint32_t w[B][4];
#pragma unroll
    for (int i = 0; i < B; ++i) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + (size_t)i * N));
        w[i][0] = v.x;
        w[i][1] = v.y;
        w[i][2] = v.z;
        w[i][3] = v.w;
    }
    const uint2 sv = __ldg(reinterpret_cast<const uint2*>(srow));
    float s[4];
    s[0] = __low2float(*reinterpret_cast<const __half2*>(&sv.x));
    s[1] = __high2float(*reinterpret_cast<const __half2*>(&sv.x));
    s[2] = __low2float(*reinterpret_cast<const __half2*>(&sv.y));
    s[3] = __high2float(*reinterpret_cast<const __half2*>(&sv.y));
    constexpr uint32_t kMask = (1u << B) - 1u;
    constexpr int kZero = 1 << (B - 1);
#pragma unroll
    for (int r = 0; r < kBlockRows; ++r) {
        const int p = r * B;
        const int wi = p >> 5, sh = p & 31;
        __half out[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            uint32_t q;
            if (sh + B <= 32) {
                q = (w[wi][c] >> sh) & kMask;
            } else {
                q = __funnelshift_r(w[wi][c], w[wi + 1 < B ? wi + 1 : wi][c], sh) & kMask;
            }
            out[c] = __float2half_rn((float)((int)q - kZero) * s[c]);
        }
        uint2 o;
        o.x = (uint32_t)__half_as_ushort(out[0]) | ((uint32_t)__half_as_ushort(out[1]) << 16);
        o.y = (uint32_t)__half_as_ushort(out[2]) | ((uint32_t)__half_as_ushort(out[3]) << 16);
        *reinterpret_cast<uint2*>(dst + (size_t)r * N) = o;
    }
}

__global__ void __launch_bounds__(128) dequant_kernel(const uint32_t* __restrict__ qw,
                                                      int64_t qw_rows,
                                                      const __half* __restrict__ scales,
                                                      const uint8_t* __restrict__ bits,
                                                      const int32_t* __restrict__ offs, int K,
                                                      int N, __half* __restrict__ w) {
    const int n = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
    const int j = blockIdx.y;
    const int nb = K / kBlockRows;
    if (n >= N) return;
    int b, off;
    if (!block_schedule_ok(bits, offs, j, nb, qw_rows, &b, &off)) {
        set_dev_error(QGEMM_DEV_BAD_SCHEDULE);
        return;
    }
    const uint32_t* src = qw + (size_t)off * N + n;
    const __half* srow = scales + (size_t)(j * kBlockRows / kGroupRows) * N + n;
    __half* dst = w + (size_t)j * kBlockRows * N + n;
    switch (b) {
        case 2: dequant_block4<2>(src, srow, dst, N); break;
        case 3: dequant_block4<3>(src, srow, dst, N); break;
        case 4: dequant_block4<4>(src, srow, dst, N); break;
        case 5: dequant_block4<5>(src, srow, dst, N); break;
        case 6: dequant_block4<6>(src, srow, dst, N); break;
        case 8: dequant_block4<8>(src, srow, dst, N); break;
        default: break;
    }
}

}  // namespace qg
