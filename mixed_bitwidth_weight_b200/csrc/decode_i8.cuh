// Byte placement of one 32-row block's codes for the integer tensor-core MMA.
//
// A block of width b is 32 codes packed LSB-first into b words per column
// (code r at stream bits [r*b, r*b + b), stream bit t = bit t%32 of word t/32).
// The integer MMA (tcgen05.mma kind::i8, K = 32) wants the block as 32
// unsigned bytes per column.  This header turns the b words into exactly eight
// 32-bit registers (32 bytes) in which every code of the block sits alone in
// one byte, at a bit offset P of that byte (P + b <= 8, P <= 6), so the byte
// reads as q * 2^P:
//   - in place: word i under a mask (2-, 4- and 8-bit blocks only need this:
//     one mask per four codes, no shift);
//   - shifted: the funnel shift by 4 of words i and i+1 under a mask (the
//     codes of 3-, 5- and 6-bit blocks that straddle a byte boundary);
//   - two sources merged: (A & mA) | (B & mB), when a register's free byte is
//     filled from a second source at the same byte position.
// The activation side (the MMA's B operand) carries, for each of the 32 byte
// slots k, the activation of the code in that slot times 2^(6 - P(k)), so
// every product is 64 * q * x whatever the width and slot.
//
// Everything here is host- and device-callable so that the placement can be
// checked on the CPU against an independent packing.
#pragma once

#include <stdint.h>

#ifdef __CUDACC__
#define QG_HD __host__ __device__ __forceinline__
#else
#define QG_HD inline
#endif

namespace qg {

// One source of a register: src 0..7 = word src in place, 8..15 = funnel
// shift by 4 of words (src - 8) and (src - 7); src < 0: unused.
struct DecSrc {
    int src;
    uint32_t mask;
};
struct DecReg {
    DecSrc a, b;
};

// Register c (0..7) of a block of width B.  The masks select, per byte, the
// field of one code; the tables were derived by enumerating which codes lie
// inside a byte of each source and pairing registers whose free bytes
// complement each other.
template <int B>
QG_HD constexpr DecReg dec_reg(int c) {
    if (B == 2) {
        const uint32_t m[4] = {0x03030303u, 0x0C0C0C0Cu, 0x30303030u, 0xC0C0C0C0u};
        return DecReg{{c >> 2, m[c & 3]}, {-1, 0u}};
    }
    if (B == 4) return DecReg{{c >> 1, (c & 1) ? 0xF0F0F0F0u : 0x0F0F0F0Fu}, {-1, 0u}};
    if (B == 8) return DecReg{{c, 0xFFFFFFFFu}, {-1, 0u}};
    if (B == 3) {
        switch (c) {
            case 0: return DecReg{{0, 0x071C0E07u}, {-1, 0u}};
            case 1: return DecReg{{0, 0x38E07038u}, {-1, 0u}};
            case 2: return DecReg{{1, 0x0E071C0Eu}, {-1, 0u}};
            case 3: return DecReg{{1, 0x7038E070u}, {-1, 0u}};
            case 4: return DecReg{{2, 0x1C0E071Cu}, {-1, 0u}};
            case 5: return DecReg{{2, 0xE07038E0u}, {-1, 0u}};
            case 6: return DecReg{{8, 0x1C00381Cu}, {9, 0x001C0000u}};
            default: return DecReg{{10, 0x00381C00u}, {9, 0x38000038u}};
        }
    }
    if (B == 5) {
        switch (c) {
            case 0: return DecReg{{2, 0x7C1FF83Eu}, {-1, 0u}};
            case 1: return DecReg{{8, 0x7C1FF83Eu}, {-1, 0u}};
            case 2: return DecReg{{0, 0x3E007C1Fu}, {4, 0x003E0000u}};
            case 3: return DecReg{{1, 0x007C1FF8u}, {4, 0xF8000000u}};
            case 4: return DecReg{{3, 0x1FF83E00u}, {4, 0x0000007Cu}};
            case 5: return DecReg{{10, 0xF83E007Cu}, {9, 0x00003E00u}};
            case 6: return DecReg{{11, 0x3E007C1Fu}, {9, 0x00F80000u}};
            default: return DecReg{{12, 0x007C1FF8u}, {9, 0x1F000000u}};
        }
    }
    // B == 6
    switch (c) {
        case 0: return DecReg{{0, 0x3FFC003Fu}, {1, 0x0000FC00u}};
        case 1: return DecReg{{2, 0xFC003FFCu}, {1, 0x003F0000u}};
        case 2: return DecReg{{3, 0x3FFC003Fu}, {4, 0x0000FC00u}};
        case 3: return DecReg{{5, 0xFC003FFCu}, {4, 0x003F0000u}};
        case 4: return DecReg{{9, 0x3FFC003Fu}, {10, 0x0000FC00u}};
        case 5: return DecReg{{8, 0xFC003FFCu}, {10, 0x003F0000u}};
        case 6: return DecReg{{12, 0x3FFC003Fu}, {13, 0x0000FC00u}};
        default: return DecReg{{11, 0xFC003FFCu}, {13, 0x003F0000u}};
    }
}

template <int B>
QG_HD uint32_t dec_source(const uint32_t* w, int src) {
    if (src < 8) return w[src];
    const int i = src - 8;
    const uint32_t hi = (i + 1 < B) ? w[i + 1] : 0u;
    return (w[i] >> 4) | (hi << 28);
}

// The eight A-operand registers of a block of width B from its B words.
template <int B>
QG_HD void decode_block_i8(const uint32_t* w, uint32_t* r) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const DecReg d = dec_reg<B>(c);
        uint32_t v = dec_source<B>(w, d.a.src) & d.a.mask;
        if (d.b.src >= 0) v |= dec_source<B>(w, d.b.src) & d.b.mask;
        r[c] = v;
    }
}

// For width B and code r (0..31): the byte slot k (register k/4, byte k%4)
// that holds it and its bit offset P there, packed as k | P << 8.  Derived
// from dec_reg: a source's byte beta under a mask field starting at bit P
// holds the code whose stream position is 32*i + shift + 8*beta + P.
template <int B>
QG_HD constexpr uint32_t dec_slot_of_code(int r) {
    for (int c = 0; c < 8; ++c) {
        const DecReg d = dec_reg<B>(c);
        for (int h = 0; h < 2; ++h) {
            const DecSrc s = h ? d.b : d.a;
            if (s.src < 0) continue;
            const int base = (s.src < 8) ? 32 * s.src : 32 * (s.src - 8) + 4;
            for (int beta = 0; beta < 4; ++beta) {
                const uint32_t byte = (s.mask >> (8 * beta)) & 0xFFu;
                if (!byte) continue;
                int P = 0;
                while (!((byte >> P) & 1u)) ++P;
                if ((base + 8 * beta + P) == r * B) return (uint32_t)(4 * c + beta) | ((uint32_t)P << 8);
            }
        }
    }
    return 0xFFFFFFFFu;  // not reached for a valid table
}

// Index of a width in {2,3,4,5,6,8}: 0..5.
QG_HD constexpr int width_index(int b) { return b == 8 ? 5 : b - 2; }

}  // namespace qg
