// Host-side probe of the tcgen05 encodings the kernels use (compiled and run
// on the CPU by test_tc_encodings.py; no GPU involved): prints the
// instruction descriptor for each "M N a_mn b_mn" given on the command line,
// then the shared-memory operand descriptors of every k-step for the tile
// heights R = 64, 128 at a few start addresses.
#include <stdio.h>
#include <stdlib.h>

#include "tc_tiles.cuh"

int main(int argc, char **argv) {
    using namespace gdn2;
    for (int i = 1; i + 3 < argc; i += 4) {
        const int M = atoi(argv[i]), N = atoi(argv[i + 1]);
        const bool a = atoi(argv[i + 2]) != 0, b = atoi(argv[i + 3]) != 0;
        printf("idesc %d %d %d %d %u\n", M, N, (int)a, (int)b, tc::idesc_bf16(M, N, a, b));
    }
    const unsigned starts[] = {0u, 1024u, 0x18400u, 0x37c00u};
    for (unsigned st : starts)
        for (int R = 64; R <= 128; R += 64)
            for (int s = 0; s < 8; ++s) {
                printf("kdesc %u %d %d %llu %u\n", st, R, s, (unsigned long long)tct::operand_desc<true>(st, R, s),
                       tct::kstep_bytes<true>(R, s));
                printf("mdesc %u %d %d %llu %u\n", st, R, s, (unsigned long long)tct::operand_desc<false>(st, R, s),
                       tct::kstep_bytes<false>(R, s));
            }
    return 0;
}
