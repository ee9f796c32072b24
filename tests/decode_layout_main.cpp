// Host driver for the decode placement check (tests/test_decode_layout.py):
// reads "b w0 .. w(b-1)" lines from stdin and prints, per line, the 32 bytes
// that the kernel's decode_block_i8<b> places in the MMA's A operand; the
// first line of output is the code -> slot table of every width.
#include <cstdio>
#include <cstdint>

#include "../mixed_bitwidth_weight_b200/csrc/decode_i8.cuh"

using namespace qg;

template <int B>
static void run(const uint32_t* w) {
    uint32_t r[8];
    decode_block_i8<B>(w, r);
    for (int k = 0; k < 32; ++k) std::printf("%u ", (r[k / 4] >> (8 * (k % 4))) & 0xFFu);
    std::printf("\n");
}

int main() {
    const int widths[6] = {2, 3, 4, 5, 6, 8};
    for (int wi = 0; wi < 6; ++wi)
        for (int r = 0; r < 32; ++r) {
            uint32_t v = 0;
            switch (widths[wi]) {
                case 2: v = dec_slot_of_code<2>(r); break;
                case 3: v = dec_slot_of_code<3>(r); break;
                case 4: v = dec_slot_of_code<4>(r); break;
                case 5: v = dec_slot_of_code<5>(r); break;
                case 6: v = dec_slot_of_code<6>(r); break;
                default: v = dec_slot_of_code<8>(r); break;
            }
            std::printf("%u ", v);
        }
    std::printf("\n");
    int b;
    while (std::scanf("%d", &b) == 1) {
        uint32_t w[8] = {0};
        for (int i = 0; i < b; ++i) std::scanf("%u", &w[i]);
        switch (b) {
            case 2: run<2>(w); break;
            case 3: run<3>(w); break;
            case 4: run<4>(w); break;
            case 5: run<5>(w); break;
            case 6: run<6>(w); break;
            case 8: run<8>(w); break;
            default: return 1;
        }
    }
    return 0;
}
