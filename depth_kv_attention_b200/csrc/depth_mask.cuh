// Column masks of one query row over a 128-column depth chunk.
//
// The depth keys of the tokens t0 .. of a query tile are rows t*Ld + i of the
// flattened [T*Ld] depth axis ("Mixture-of-Depths Attention", gist.science
// German summary §2: depth KV laid out along one T x L axis); a row sees only
// the Ld rows of its own token (mhpn.cn §2.2, the same-token half of the dual
// mask), and with a per-token selection only the slots the token selects
// (gist.science German summary §5: bounded depth-KV slots).
#pragma once

#include <cstdint>

namespace moda {

// Mask of the selectable slots 0 .. Ld-1 (Ld <= 64).
__device__ __forceinline__ unsigned long long depth_slot_bits(int Ld) {
    return Ld >= 64 ? ~0ull : ((1ull << Ld) - 1ull);
}

// Visible columns of a row whose own depth rows start at chunk column `lo`
// (negative or >= 128 when they begin before or after the chunk) and span Ld
// columns, as four words: bit k of w[c] = column 32c + k. With `has_sel`,
// `sel` (bits >= Ld clear) keeps only the selected slots.
__device__ __forceinline__ void depth_col_mask(int lo, int Ld, bool has_sel,
                                               unsigned long long sel, uint32_t (&w)[4]) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int sh = lo - 32 * c;  // column 32c + k holds slot k - sh
        if (has_sel) {
            uint32_t v = 0;
            if (sh >= 0 && sh < 32) v = (uint32_t)(sel << sh);
            else if (sh < 0 && sh > -64) v = (uint32_t)(sel >> (-sh));
            w[c] = v;
        } else {
            const int a = min(max(sh, 0), 32), e = min(max(sh + Ld, 0), 32);  // bits [a, e)
            const uint32_t below_e = e >= 32 ? 0xffffffffu : ((1u << e) - 1u);
            const uint32_t below_a = a >= 32 ? 0xffffffffu : ((1u << a) - 1u);
            w[c] = below_e & ~below_a;
        }
    }
}

}  // namespace moda
