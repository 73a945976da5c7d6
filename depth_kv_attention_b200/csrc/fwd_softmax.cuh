// One key item of the forward's online softmax for one query row (one
// thread = one TMEM lane), shared by the single-CTA and the CTA-pair forward
// kernels.
//
// What it computes: "动态混合深度注意力机制MoDA技术解析" (mhpn.cn) §2.2, the
// online-softmax state (running max m, running sum "acc" = l, output o)
// carried across key blocks, with the dual mask (causal over the sequence,
// same position over depth); §1.2, one softmax over sequence and depth logits
// scaled by 1/sqrt(d) (sl2 = scale * log2 e: logits in the log2 domain).
//
// The item's S (128 fp32 columns) is read from TMEM, masked, its row max
// folded into m with lazy rescaling (the exponent reference moves only when a
// row max exceeds it by 2^8; O and l are then rescaled together, so O / l is
// exact), P = 2^(S*sl2 - m) written back in bf16 over the first 64 columns of
// S (the A operand of O += P V) and added into l. Returns once P is in TMEM
// and fenced for the thread synchronisation that publishes it.
#pragma once

#include <cmath>
#include <cstdint>

#include "depth_mask.cuh"
#include "sm100_ptx.cuh"

namespace moda {

constexpr float kRescaleThreshold = 8.0f;  // log2 units

// Of every 8 column pairs of a row, pairs kPolyFrom..7 take exp2 from the
// FMA-pipe polynomial, the rest from the MUFU unit (which alone would be
// as busy as the tensor core at d = 128).
#ifndef MODA_POLY_FROM
#define MODA_POLY_FROM 8
#endif
constexpr int kPolyFrom = MODA_POLY_FROM;

// seq_item: a causal sequence tile whose first key is kbase (row token t);
// otherwise a depth chunk in which this row's own depth columns start at
// dep_lo (negative or >= 128 when they begin before or after the chunk).
// it: items this row has taken part in before (0 = O holds nothing yet).
__device__ __forceinline__ void softmax_item(uint32_t tS, uint32_t tO, bool seq_item, int kbase, int t,
                                             int dep_lo, int Ld, bool has_sel, unsigned long long sel,
                                             float sl2, int it, float& m, float& l) {
    float s[128];
    {
        uint32_t su[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) ptx::tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&su[c * 32]));
        ptx::tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(su[c]);
    }
    if (seq_item) {
        if (kbase + 127 > t) {
#pragma unroll
            for (int c = 0; c < 128; ++c)
                if (kbase + c > t) s[c] = -INFINITY;
        }
    } else {
        // same-token mask: this row's depth columns (selected slots only)
        uint32_t vis[4];
        depth_col_mask(dep_lo, Ld, has_sel, sel, vis);
#pragma unroll
        for (int c = 0; c < 128; ++c)
            if (!((vis[c >> 5] >> (c & 31)) & 1u)) s[c] = -INFINITY;
    }
    float mx;
    {
        float mp[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mp[e] = ptx::max3(s[e], s[8 + e], s[16 + e]);
#pragma unroll
        for (int c = 24; c < 120; c += 16)
#pragma unroll
            for (int e = 0; e < 8; ++e) mp[e] = ptx::max3(mp[e], s[c + e], s[c + 8 + e]);
#pragma unroll
        for (int e = 0; e < 8; ++e) mp[e] = fmaxf(mp[e], s[120 + e]);
        mx = ptx::max3(ptx::max3(mp[0], mp[1], mp[2]), ptx::max3(mp[3], mp[4], mp[5]), fmaxf(mp[6], mp[7]));
    }
    const float mxs = mx * sl2;
    // tcgen05.ld / st are warp-collective: the rescale decision is made
    // warp-uniform.
    if (__any_sync(0xffffffffu, mxs > m + kRescaleThreshold)) {
        // Move the exponent reference of every row of the warp to its running
        // max; rescale l and the O already accumulated (every earlier P V has
        // completed: S of this item was committed after it).
        const float mnew = fmaxf(m, mxs);
        const float corr = (mnew == -INFINITY) ? 1.f : ptx::ex2(m - mnew);
        if (it > 0) {
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t o[32];
                ptx::tmem_ld32(tO + c * 32, o);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * corr);
                ptx::tmem_st32(tO + c * 32, o);
            }
        }
        l *= corr;
        m = mnew;
    }
    const float mref = (m == -INFINITY) ? 0.f : m;
    const float2 sl2x2 = make_float2(sl2, sl2), nm2 = make_float2(-mref, -mref);
    float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
    uint32_t pk[64];
#pragma unroll
    for (int c = 0; c < 64; ++c) {
        const float2 xv = ptx::fma2(make_float2(s[2 * c], s[2 * c + 1]), sl2x2, nm2);
        float2 pv;
        if ((c & 7) >= kPolyFrom) {
            pv = ptx::exp2_poly2(xv);  // FMA pipe
        } else {
            pv.x = ptx::ex2(xv.x);     // MUFU
            pv.y = ptx::ex2(xv.y);
        }
        acc[c & 3] = ptx::add2(acc[c & 3], pv);
        pk[c] = ptx::pack_bf16x2(pv.x, pv.y);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) ptx::tmem_st16(tS + q * 16, *reinterpret_cast<uint32_t(*)[16]>(&pk[q * 16]));
    ptx::tmem_wait_st();
    ptx::tc_fence_before();
    {
        const float2 a01 = ptx::add2(acc[0], acc[1]), a23 = ptx::add2(acc[2], acc[3]);
        const float2 a = ptx::add2(a01, a23);
        l += a.x + a.y;
    }
}

}  // namespace moda
