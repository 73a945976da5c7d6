// Tensor-core MoDA forward for sm_100a: TMA -> shared memory -> tcgen05.mma
// -> TMEM, with the online softmax on the CUDA cores.
//
// What it computes: "动态混合深度注意力机制MoDA技术解析" (mhpn.cn) §1.2, one softmax
// over [Q K_l^T || Q K_depth^T] / sqrt(d) times [V_l || V_depth]; §2.2, the
// online-softmax state (running max m, running sum "acc" = l, output o)
// carried across key blocks, with the dual mask (causal over the sequence,
// same position over depth).
//
// How (B200 design, not the pages' kernel):
//  * Work unit = (b, kv-head, block of 2n tokens), n = 128 / G. It holds two
//    128-row query tiles; a row is (token, head) in token-major order
//    (row = token * G + head), so one query tile covers the G heads of a GQA
//    group for n tokens and every K/V tile is shared by all of them
//    ("Mixture-of-Depths Attention", gist.science German summary §2,
//    group-aware indexing).
//  * Key items: the causal sequence tiles of 128 keys, then the depth chunks.
//    The depth keys of the unit's tokens are rows t0*Ld .. (t0+2n)*Ld of the
//    native [B, T*Ld, Hkv, d] view of kd (the flattened T x L axis of the
//    same summary's flash-compatible layout), loaded 128 rows at a time by
//    TMA and masked to the row's own token (chunk-aware: only the unit's own
//    depth range is read). Each depth row is read once per unit.
//  * Warp roles: warps 0-3 and 4-7 run the softmax of query tiles 0 and 1
//    (one thread per row, TMEM lane = row); warp 8 issues TMA loads into a
//    5-stage ring; lane 0 of warp 9 issues every tcgen05.mma (warps 10-11
//    only pad the third warpgroup for the register reallocation).
//    TMEM: S0 | S1 | O0 | O1, 128
//    fp32 columns each; P (bf16) overwrites the first 64 columns of S and is
//    the TMEM A operand of O += P V. While tile 0's softmax runs, the tensor
//    core computes tile 1's S, and the other way round.
//  * Lazy rescaling: the running max used as the exponent reference only
//    moves when a new row max exceeds it by more than 2^8; O and l use the
//    same reference, so the final O / l is exact.
//  * Every mbarrier wait is bounded. On expiry the CTA records
//    MODA_ERR_DEVICE_TIMEOUT in the device status word, drains its own TMA
//    loads and MMAs, frees TMEM and exits.
#include <cuda_bf16.h>

#include <cmath>
#include <cstring>

#include "depth_mask.cuh"
#include "fwd_softmax.cuh"
#include "moda_internal.h"
#include "sm100_ptx.cuh"
#include "tmap_host.h"

namespace moda {
namespace {

constexpr int kD = 128;                // head dim
constexpr int kBM = 128;               // rows per query tile
constexpr int kBN = 128;               // keys per item
constexpr int kStages = 5;             // K/V ring depth (one tile per stage)
constexpr int kTileBytes = kBM * kD * 2;       // 32 KB
constexpr int kHalfBytes = kTileBytes / 2;     // one 64-column swizzled half
// 3 warpgroups: two softmax warpgroups (one per query tile) and one for the
// TMA producer warp, the MMA warp and two idle warps. Registers at launch:
// 384 x 168; after reallocation 2 x 128 x 216 + 128 x 72 = 384 x 168.
constexpr int kThreads = 384;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kSoftmaxRegs = 216;
constexpr int kControlRegs = 72;
constexpr uint32_t kNoPollLimit = 0;  // drains: time bound only

struct TcFwdParams {
    CUtensorMap tm_q, tm_k, tm_v, tm_kd, tm_vd;
    void* out;
    float* lse;
    int B, T, Hq, Hkv, G, n, Ld, nblk;
    int tb_lo, nblk_q;  // token blocks tb_lo .. tb_lo + nblk_q - 1 of each (b, kv-head) in this launch
    float sl2;  // scale * log2(e)
    int depth_packed;
    const unsigned long long* depth_sel;  // [B,T] slot masks or null
    const float* kd_scale;  // 8-bit depth: [B,T,Ld,Hkv] row scales (tm_kd / tm_vd map int8 codes)
    const float* vd_scale;
    unsigned int* status;
    unsigned int wait_limit;
};

struct __align__(8) Bars {
    uint64_t q_full;
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t raw_full[kStages];  // 8-bit depth tile landed (before dequantisation)
    uint64_t s_full[2];
    uint64_t p_full[2];
    uint64_t o_final[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};

constexpr int kSmemBytes = 2 * kTileBytes + kStages * kTileBytes + 1024 /*bars*/ + 1024 /*align*/;
static_assert(kSmemBytes <= 232448, "shared memory per CTA");
static_assert(sizeof(Bars) <= 1024, "barrier block");

__device__ __forceinline__ void flag_timeout(TcFwdParams const& p, Bars* bars) {
    *reinterpret_cast<volatile int*>(&bars->abort_flag) = 1;
    atomicOr(p.status, 1u);
}

// Ring use index of depth tile `seq` in stage `st`: how many earlier depth
// tiles (sequence numbers >= first) used the same stage. Its parity is the
// phase of raw_full[st] that marks this tile's arrival.
__device__ __forceinline__ uint32_t depth_use(int seq, int first) {
    const int st = seq % kStages;
    const int f = first + ((st - first % kStages) + kStages) % kStages;
    return (uint32_t)((seq - f) / kStages);
}

// 8-bit depth tiles: the producer's TMA puts a tile of 128 rows x 128 int8
// codes as plain 128-byte lines into the second half of its ring slot; warps
// 10 and 11 dequantise it in place into the bf16 128B-swizzled K-major layout
// the MMA reads (row r: features 0-63 at r*128 of the first half, 64-127 at
// r*128 of the second, 16-byte chunk j stored at chunk j ^ (r % 8)). A row's
// second-half output overlaps only its own source line: each thread converts
// its row in two passes, features 0-63 (written to the first half, which
// holds no source) and then 64-127, whose source it reads before writing.
// value = fp32(code * scale) rounded to bf16.
__device__ __forceinline__ void dequant_row_q8(uint8_t* slot, int r, float sigma) {
    const uint4* src = reinterpret_cast<const uint4*>(slot + kHalfBytes + r * 128);
    const float2 bias = make_float2(-8388736.f, -8388736.f);  // 2^23 + 128
    const float2 sg = make_float2(sigma, sigma);
#pragma unroll
    for (int pass = 0; pass < 2; ++pass) {
    uint4 in[4];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) in[jj] = src[4 * pass + jj];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
        const int j = 4 * pass + jj;
        const uint32_t w4[4] = {in[jj].x ^ 0x80808080u, in[jj].y ^ 0x80808080u, in[jj].z ^ 0x80808080u,
                                in[jj].w ^ 0x80808080u};
        uint32_t o[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            // code + 128 into the low byte of 2^23: the float 2^23 + code + 128
            const float2 lo = make_float2(__uint_as_float(__byte_perm(w4[q], 0x4B000000u, 0x7540)),
                                          __uint_as_float(__byte_perm(w4[q], 0x4B000000u, 0x7541)));
            const float2 hi = make_float2(__uint_as_float(__byte_perm(w4[q], 0x4B000000u, 0x7542)),
                                          __uint_as_float(__byte_perm(w4[q], 0x4B000000u, 0x7543)));
            const float2 a = ptx::mul2(ptx::add2(lo, bias), sg);
            const float2 b = ptx::mul2(ptx::add2(hi, bias), sg);
            o[2 * q] = ptx::pack_bf16x2(a.x, a.y);
            o[2 * q + 1] = ptx::pack_bf16x2(b.x, b.y);
        }
        // features 16j .. 16j+15 = output chunks 2j, 2j+1 (8 features each)
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int oc = 2 * j + u, h = oc >> 3, cj = oc & 7;
            uint4* dst = reinterpret_cast<uint4*>(slot + h * kHalfBytes + r * 128 + ((cj ^ (r & 7)) << 4));
            *dst = make_uint4(o[4 * u], o[4 * u + 1], o[4 * u + 2], o[4 * u + 3]);
        }
    }
    }
}

template <bool kQ8>
__global__ void __launch_bounds__(kThreads, 1) moda_fwd_tc_kernel(const __grid_constant__ TcFwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;                                // 2 tiles
    uint8_t* sRing = smem + 2 * kTileBytes;            // kStages tiles
    Bars* bars = reinterpret_cast<Bars*>(sRing + kStages * kTileBytes);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const uint32_t wait_limit = p.wait_limit;  // 0: time bound only
    volatile int* abort_flag = &bars->abort_flag;

    // ---- work unit: (b, kv-head)-major, heaviest (latest) token blocks
    // first within each. CTAs in flight then share one kv-head's K/V stream
    // in L2 (at T = 64K one head's K + V is 32 MB; all four heads' streams
    // together exceed the 126 MB L2), and the lightest blocks come last.
    const int bh = blockIdx.x / p.nblk_q;
    const int tb = p.tb_lo + p.nblk_q - 1 - blockIdx.x % p.nblk_q;
    const int b = bh / p.Hkv, kvh = bh % p.Hkv;
    const int n = p.n;
    const int t0 = tb * 2 * n;
    // Items: the causal sequence tiles of 128 keys, then the depth chunks:
    // 128-row slices of the unit's depth rows t0*Ld .. (t0+2n)*Ld of the
    // [B, T*Ld, Hkv, d] view. Every item occupies two ring slots (K, V).
    int n_kv[2], nv[2];
    for (int i = 0; i < 2; ++i) {
        const int last = min(p.T - 1, t0 + (i + 1) * n - 1);
        n_kv[i] = last / kBN + 1;
        nv[i] = max(0, min(n, p.T - t0 - i * n));  // tokens of tile i inside the sequence
    }
    const int n_seq = n_kv[1];
    const int n_dep = ((nv[0] + nv[1]) * p.Ld + kBN - 1) / kBN;
    const int n_items = n_seq + n_dep;
    // Tile i takes part in sequence items up to its last token's tile, and in
    // the depth chunks that overlap its own tokens' depth rows.
    // (selects rather than indexing, so that a runtime tile index keeps the
    // arrays in registers)
    // Depth chunks [dlo_i, dhi_i) (as item indices) overlap tile i's rows
    // i*n*Ld .. (i*n + nv_i)*Ld.
    int dlo[2], dhi[2];
    for (int i = 0; i < 2; ++i) {
        const int row0 = i * n * p.Ld, row1 = row0 + nv[i] * p.Ld;
        dlo[i] = n_seq + row0 / kBN;
        dhi[i] = nv[i] > 0 ? n_seq + (row1 + kBN - 1) / kBN : dlo[i];
    }
    auto part = [&](int i, int x) {
        return x < (i ? n_kv[1] : n_kv[0]) || (x >= (i ? dlo[1] : dlo[0]) && x < (i ? dhi[1] : dhi[0]));
    };

    if (threadIdx.x == 0) {
        ptx::mbar_init(&bars->q_full, 1);
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(&bars->full[s], 1);
            ptx::mbar_init(&bars->empty[s], 1);
            ptx::mbar_init(&bars->raw_full[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&bars->s_full[i], 1);
            ptx::mbar_init(&bars->p_full[i], 4);  // one arrival per warp
            ptx::mbar_init(&bars->o_final[i], 1);
        }
        ptx::mbar_init(&bars->drain, 1);
        bars->abort_flag = 0;
        ptx::fence_barrier_init();
        ptx::fence_proxy_async_smem();
    }
    if (warp == 0) {
        ptx::tmem_alloc(&bars->tmem_base, 512);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    // Register reallocation happens inside each role's branch, so that every
    // instruction of a role is compiled under that role's register budget.
    if (warp >= 8) ptx::setmaxnreg_dec<kControlRegs>();
    if (warp == kProducerWarp) {
        // The whole warp runs the schedule (its values stay warp-uniform);
        // lane 0 issues the copies.
        const uint32_t lead = lane == 0;
        if (lead) {
            ptx::prefetch_tmap(&p.tm_q);
            ptx::prefetch_tmap(&p.tm_k);
            ptx::prefetch_tmap(&p.tm_v);
            if (p.Ld > 0) {
                ptx::prefetch_tmap(&p.tm_kd);
                ptx::prefetch_tmap(&p.tm_vd);
            }
        }
        ptx::mbar_arrive_expect_tx_lead(&bars->q_full, 2 * kTileBytes, lead);
        for (int i = 0; i < 2; ++i)
            for (int hf = 0; hf < 2; ++hf)
                ptx::tma_load_4d_lead(sQ + i * kTileBytes + hf * kHalfBytes, &p.tm_q, &bars->q_full, hf * 64,
                                      kvh * p.G, t0 + i * n, b, lead);
        int seq = 0;
        bool ok = true;
        for (int x = 0; x < n_items && ok; ++x) {
            for (int kv = 0; kv < 2; ++kv, ++seq) {
                const int st = seq % kStages;
                const uint32_t ph = (seq / kStages) & 1;
                if (!__all_sync(0xffffffffu, ptx::mbar_wait(&bars->empty[st], ph ^ 1, wait_limit, abort_flag))) {
                    if (lead) flag_timeout(p, bars);
                    ok = false;
                    break;
                }
                uint8_t* dst = sRing + st * kTileBytes;
                if (kQ8 && x >= n_seq) {
                    // int8 codes into the slot's second half; warps 10-11
                    // dequantise them and complete full[st]
                    ptx::mbar_arrive_expect_tx_lead(&bars->raw_full[st], kHalfBytes, lead);
                    ptx::tma_load_4d_lead(dst + kHalfBytes, kv ? &p.tm_vd : &p.tm_kd, &bars->raw_full[st], 0, kvh,
                                          t0 * p.Ld + (x - n_seq) * kBN, b, lead);
                    continue;
                }
                ptx::mbar_arrive_expect_tx_lead(&bars->full[st], kTileBytes, lead);
                for (int hf = 0; hf < 2; ++hf) {
                    if (x < n_seq) {
                        ptx::tma_load_4d_lead(dst + hf * kHalfBytes, kv ? &p.tm_v : &p.tm_k, &bars->full[st], hf * 64,
                                              kvh, x * kBN, b, lead);
                    } else {
                        const int row = t0 * p.Ld + (x - n_seq) * kBN;
                        const CUtensorMap* m = kv ? &p.tm_vd : &p.tm_kd;
                        if (p.depth_packed)
                            ptx::tma_load_4d_lead(dst + hf * kHalfBytes, m, &bars->full[st], hf * 64, row, kvh, b, lead);
                        else
                            ptx::tma_load_4d_lead(dst + hf * kHalfBytes, m, &bars->full[st], hf * 64, kvh, row, b, lead);
                    }
                }
            }
        }
        // Drain: every load this CTA issued lands before the CTA can exit.
        ptx::mbar_wait(&bars->q_full, 0, kNoPollLimit, nullptr);
        for (int s = (seq > kStages ? seq - kStages : 0); s < seq; ++s) {
            if (kQ8 && s >= 2 * n_seq)
                ptx::mbar_wait(&bars->raw_full[s % kStages], depth_use(s, 2 * n_seq) & 1, kNoPollLimit, nullptr);
            else
                ptx::mbar_wait(&bars->full[s % kStages], (s / kStages) & 1, kNoPollLimit, nullptr);
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // One thread runs the MMA schedule: a tcgen05.mma issued by a single
        // thread costs about 60 cycles, against 80-90 when the whole warp
        // executes it predicated on one lane (measured on the B200), and the
        // tensor core finishes a 128x128x16 MMA in 64 cycles, so only the
        // single-thread form keeps it fed. Descriptors are formed once per
        // tile; a K step only adds a constant to the 14-bit address field
        // (K-major: 32 B per 16 columns within a 128-byte row, 16 KB per
        // 64-column half; MN-major: 16 rows of 128 B = 2048 B).
        if (lane == 0) {
            constexpr uint32_t idesc_qk = ptx::idesc_bf16_f32(kBM, kBN, 0, 0);
            constexpr uint32_t idesc_pv = ptx::idesc_bf16_f32(kBM, kD, 0, 1);
            const uint32_t sQa = ptx::smem_u32(sQ);
            const uint32_t sRa = ptx::smem_u32(sRing);
            uint64_t dq_desc[2];
            for (int i = 0; i < 2; ++i) dq_desc[i] = ptx::umma_desc_sw128(sQa + i * kTileBytes, 16, 1024);
            // ring slot st's K / V descriptors: the stage's offset added to the
            // 14-bit address field of slot 0's (addresses stay below 2^18 B)
            const uint64_t k0 = ptx::umma_desc_sw128(sRa, 16, 1024);
            const uint64_t v0 = ptx::umma_desc_sw128(sRa, kHalfBytes, 1024);
            constexpr uint64_t kSlotUnits = kTileBytes >> 4;
            // (a plain bounded wait: one thread, no warp vote)
            auto wait_all = [&](uint64_t* bar, uint32_t parity) {
                return ptx::mbar_wait(bar, parity, wait_limit, abort_flag);
            };
            bool ok = wait_all(&bars->q_full, 0);
            if (!ok) flag_timeout(p, bars);
            ptx::tc_fence_after();
            int cnt_p0 = 0, cnt_p1 = 0;
            // ring position of the V tile of item x (2x + 1) and of the K tile of
            // item x + 1 (2x + 2) as (stage, phase), advanced without divisions
            int st_v = 1, ph_v = 0;
            auto advance = [](int& st, int& ph) {
                if (++st == kStages) {
                    st = 0;
                    ph ^= 1;
                }
            };
            // S_i = Q_i K^T for the K tile in ring stage ST
#define MODA_ISSUE_S(I, ST)                                                                    \
    do {                                                                                       \
        const uint64_t kd_ = k0 + (uint64_t)(ST) * kSlotUnits;                                 \
        const uint64_t qd_ = dq_desc[I];                                                       \
        _Pragma("unroll") for (int k = 0; k < kD / 16; ++k) {                                  \
            const uint64_t off = (uint64_t)((k >> 2) * (kHalfBytes >> 4) + (k & 3) * 2);        \
            ptx::mma_ss(tmem + (I) * 128, qd_ + off, kd_ + off, idesc_qk, k > 0);   \
        }                                                                                      \
        ptx::mma_commit(&bars->s_full[I]);                                          \
    } while (0)
            if (ok) ok = wait_all(&bars->full[0], 0);
            if (!ok) flag_timeout(p, bars);
            ptx::tc_fence_after();
            if (ok) {
                if (part(0, 0)) MODA_ISSUE_S(0, 0);
                if (part(1, 0)) MODA_ISSUE_S(1, 0);
                ptx::mma_commit(&bars->empty[0]);
            }
            for (int x = 0; x < n_items && ok; ++x) {
                int st_k = st_v, ph_k = ph_v;
                advance(st_k, ph_k);
                const bool next = x + 1 < n_items;
                ok = wait_all(&bars->full[st_v], ph_v);
                if (!ok) {
                    flag_timeout(p, bars);
                    break;
                }
                ptx::tc_fence_after();
                const uint64_t vd = v0 + (uint64_t)st_v * kSlotUnits;
                bool k_ready = false;
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    if (!ok) break;
                    if (part(i, x)) {
                        // O_i += P_i V once the softmax has published P_i
                        const int cnt = i ? cnt_p1 : cnt_p0;
                        if (!wait_all(&bars->p_full[i], cnt & 1)) {
                            flag_timeout(p, bars);
                            ok = false;
                            break;
                        }
                        ptx::tc_fence_after();
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            ptx::mma_ts(tmem + 256 + i * 128, tmem + i * 128 + k * 8, vd + (uint64_t)(k * 128),
                                        idesc_pv, (cnt > 0 || k > 0) ? 1u : 0u);
                        if (i) ++cnt_p1; else ++cnt_p0;
                    }
                    if (next && part(i, x + 1)) {
                        if (!k_ready) {
                            if (!wait_all(&bars->full[st_k], ph_k)) {
                                flag_timeout(p, bars);
                                ok = false;
                                break;
                            }
                            ptx::tc_fence_after();
                            k_ready = true;
                        }
                        MODA_ISSUE_S(i, st_k);
                    }
                }
                if (!ok) break;
                ptx::mma_commit(&bars->empty[st_v]);
                if (next) ptx::mma_commit(&bars->empty[st_k]);
                st_v = st_k;
                ph_v = ph_k;
                advance(st_v, ph_v);
            }
#undef MODA_ISSUE_S
            if (ok) {
                ptx::mma_commit(&bars->o_final[0]);
                ptx::mma_commit(&bars->o_final[1]);
            }
            // Drain: all MMAs issued by this thread complete before TMEM is freed.
            ptx::mma_commit(&bars->drain);
            ptx::mbar_wait(&bars->drain, 0, kNoPollLimit, nullptr);
        }
        __syncwarp();
    } else if (kQ8 && warp >= 10) {
        // ------------------------------------ 8-bit depth: dequantisation
        const int ct = threadIdx.x - 10 * 32;  // 0..63: rows ct and ct + 64
        const long long srow0 = (long long)b * p.T * p.Ld;
        for (int x = n_seq; x < n_items; ++x) {
            const int row0 = t0 * p.Ld + (x - n_seq) * kBN;  // first depth row of the tile
            for (int kv = 0; kv < 2; ++kv) {
                const int seq = 2 * x + kv, st = seq % kStages;
                const float* scl = kv ? p.vd_scale : p.kd_scale;
                float sg[2];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int row = row0 + ct + 64 * u;
                    sg[u] = row < p.T * p.Ld ? __ldg(scl + (srow0 + row) * p.Hkv + kvh) : 0.f;
                }
                const bool got = ptx::mbar_wait(&bars->raw_full[st], depth_use(seq, 2 * n_seq) & 1, wait_limit,
                                                abort_flag);
                if (!ptx::bar_and(1, 64, got)) {
                    if (ct == 0) flag_timeout(p, bars);
                    x = n_items;
                    break;
                }
                uint8_t* slot = sRing + st * kTileBytes;
                dequant_row_q8(slot, ct, sg[0]);
                dequant_row_q8(slot, ct + 64, sg[1]);
                ptx::fence_proxy_async_smem();  // generic-proxy writes -> tensor core
                ptx::bar_sync(1, 64);
                if (ct == 0) ptx::mbar_arrive(&bars->full[st]);
            }
        }
    } else if (warp < 8) {
        // ------------------------------------------------ softmax warpgroups
        ptx::setmaxnreg_inc<kSoftmaxRegs>();
        const int i = warp / 4;            // query tile
        const int r = (warp % 4) * 32 + lane;  // row = TMEM lane
        const uint32_t lane_off = (uint32_t)((warp % 4) * 32) << 16;
        const uint32_t tS = tmem + lane_off + i * 128;
        const uint32_t tO = tmem + lane_off + 256 + i * 128;
        const int tl = i * n + r / p.G;    // token offset in the unit
        const int t = t0 + tl;
        const int h = kvh * p.G + r % p.G;
        const float sl2 = p.sl2;
        const bool has_sel = p.depth_sel != nullptr;
        const unsigned long long sel =
            has_sel && t < p.T ? p.depth_sel[(long long)b * p.T + t] & depth_slot_bits(p.Ld) : 0ull;
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        int it = 0;                        // items this tile has taken part in
        for (int x = 0; x < n_items; ++x) {
            if (!part(i, x)) continue;
            // tcgen05.ld / st below are warp-collective: every decision that
            // guards them is made warp-uniform.
            const bool got = ptx::mbar_wait(&bars->s_full[i], it & 1, wait_limit, abort_flag);
            if (!__all_sync(0xffffffffu, got)) {
                flag_timeout(p, bars);
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            softmax_item(tS, tO, x < n_seq, x * kBN, t, tl * p.Ld - (x - n_seq) * kBN, p.Ld, has_sel, sel, sl2,
                         it, m, l);
            // one arrival per warp: 128 per-thread arrivals on one barrier
            // word serialise on the tile's critical chain
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&bars->p_full[i]);
            ++it;
        }
        if (ok) {
            const bool got = ptx::mbar_wait(&bars->o_final[i], 0, wait_limit, abort_flag);
            if (!__all_sync(0xffffffffu, got)) {
                flag_timeout(p, bars);
                ok = false;
            }
        }
        ptx::tc_fence_after();
        if (ok) {
            const bool valid = t < p.T;
            const float inv = 1.f / l;
            __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.out) + (((long long)b * p.T + (valid ? t : 0)) * p.Hq + h) * kD;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t o[32];
                ptx::tmem_ld32(tO + c * 32, o);
                ptx::tmem_wait_ld();
                uint32_t w[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    w[e] = ptx::pack_bf16x2(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
                if (valid) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
                    for (int v = 0; v < 4; ++v) dst[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
                }
            }
            if (valid && p.lse)
                p.lse[((long long)b * p.Hq + h) * p.T + t] = (m + __log2f(l)) * 0.6931471805599453f;
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 512);
    }
}

__global__ void exp2_poly_kernel(const float* x, float* y, int n) {
    const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (i + 1 < n) {
        const float2 r = ptx::exp2_poly2(make_float2(x[i], x[i + 1]));
        y[i] = r.x;
        y[i + 1] = r.y;
    } else if (i < n) {
        y[i] = ptx::exp2_poly2(make_float2(x[i], 0.f)).x;
    }
}

}  // namespace

cudaError_t launch_exp2_poly(const float* x, float* y, int n, cudaStream_t s) {
    const int pairs = (n + 1) / 2;
    exp2_poly_kernel<<<(pairs + 255) / 256, 256, 0, s>>>(x, y, n);
    return cudaGetLastError();
}

bool fwd_tc_supported(const FwdArgs& a) {
    if (a.dtype != MODA_BF16 || a.d != kD) return false;
    if (a.G < 1 || a.G > 128 || 128 % a.G) return false;
    // natural q / k / v / out strides (the ABI's layouts)
    const Strides4 sq = strides_q(a.T, a.Hq, a.d), skv = strides_q(a.T, a.Hkv, a.d);
    if (a.sq.sb != sq.sb || a.sq.st != sq.st || a.sq.sh != sq.sh) return false;
    if (a.so.sb != sq.sb || a.so.st != sq.st || a.so.sh != sq.sh) return false;
    if (a.skv.sb != skv.sb || a.skv.st != skv.st || a.skv.sh != skv.sh) return false;
    if ((long long)a.T * a.Ld >= (1LL << 31)) return false;  // TMA coordinates are int32
    return true;
}

cudaError_t launch_fwd_tc(const FwdArgs& a, cudaStream_t s) {
    TcFwdParams p;
    memset(&p, 0, sizeof(p));
    const int G = a.G, n = 128 / G;
    const cuuint64_t e = 2;  // bytes per bf16
    {
        const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)a.Hq, (cuuint64_t)a.T, (cuuint64_t)a.B};
        const cuuint64_t st[3] = {kD * e, (cuuint64_t)a.Hq * kD * e, (cuuint64_t)a.T * a.Hq * kD * e};
        const cuuint32_t box[4] = {64, (cuuint32_t)G, (cuuint32_t)n, 1};
        if (!make_tmap_bf16_4d(&p.tm_q, a.q, dims, st, box)) return cudaErrorInvalidValue;
    }
    {
        const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)a.Hkv, (cuuint64_t)a.T, (cuuint64_t)a.B};
        const cuuint64_t st[3] = {kD * e, (cuuint64_t)a.Hkv * kD * e, (cuuint64_t)a.T * a.Hkv * kD * e};
        const cuuint32_t box[4] = {64, 1, (cuuint32_t)kBN, 1};
        if (!make_tmap_bf16_4d(&p.tm_k, a.k, dims, st, box)) return cudaErrorInvalidValue;
        if (!make_tmap_bf16_4d(&p.tm_v, a.v, dims, st, box)) return cudaErrorInvalidValue;
    }
    const bool packed = a.Ld > 0 && !a.depth_q8 && a.sdep.si == kD;  // [B, Hkv, T*Ld, d]
    if (a.Ld > 0 && a.depth_q8) {
        // int8 codes, [B, T*Ld, Hkv, 128] bytes
        const cuuint64_t rows = (cuuint64_t)a.T * a.Ld;
        const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)a.Hkv, rows, (cuuint64_t)a.B};
        const cuuint64_t st[3] = {(cuuint64_t)kD, (cuuint64_t)a.Hkv * kD, rows * a.Hkv * kD};
        const cuuint32_t box[4] = {(cuuint32_t)kD, 1, (cuuint32_t)kBN, 1};
        if (!make_tmap_u8_4d(&p.tm_kd, a.kd, dims, st, box)) return cudaErrorInvalidValue;
        if (!make_tmap_u8_4d(&p.tm_vd, a.vd, dims, st, box)) return cudaErrorInvalidValue;
    } else if (a.Ld > 0) {
        const cuuint64_t rows = (cuuint64_t)a.T * a.Ld;
        if (packed) {
            const cuuint64_t dims[4] = {(cuuint64_t)kD, rows, (cuuint64_t)a.Hkv, (cuuint64_t)a.B};
            const cuuint64_t st[3] = {kD * e, rows * kD * e, (cuuint64_t)a.Hkv * rows * kD * e};
            const cuuint32_t box[4] = {64, (cuuint32_t)kBN, 1, 1};
            if (!make_tmap_bf16_4d(&p.tm_kd, a.kd, dims, st, box)) return cudaErrorInvalidValue;
            if (!make_tmap_bf16_4d(&p.tm_vd, a.vd, dims, st, box)) return cudaErrorInvalidValue;
        } else {
            const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)a.Hkv, rows, (cuuint64_t)a.B};
            const cuuint64_t st[3] = {kD * e, (cuuint64_t)a.Hkv * kD * e, rows * a.Hkv * kD * e};
            const cuuint32_t box[4] = {64, 1, (cuuint32_t)kBN, 1};
            if (!make_tmap_bf16_4d(&p.tm_kd, a.kd, dims, st, box)) return cudaErrorInvalidValue;
            if (!make_tmap_bf16_4d(&p.tm_vd, a.vd, dims, st, box)) return cudaErrorInvalidValue;
        }
    } else {
        p.tm_kd = p.tm_k;
        p.tm_vd = p.tm_v;
    }
    p.out = a.out;
    p.lse = a.lse;
    p.B = a.B; p.T = a.T; p.Hq = a.Hq; p.Hkv = a.Hkv; p.G = G; p.n = n; p.Ld = a.Ld;
    p.nblk = (a.T + 2 * n - 1) / (2 * n);
    // query-token range of this launch, in whole units of 2n tokens
    if (a.q_tok0 % (2 * n) != 0 || a.q_tok0 < 0 || a.q_tok1 < 0 || a.q_tok1 > a.T) return cudaErrorInvalidValue;
    p.tb_lo = a.q_tok0 / (2 * n);
    const int tb_hi = a.q_tok1 ? (a.q_tok1 + 2 * n - 1) / (2 * n) : p.nblk;
    p.nblk_q = tb_hi - p.tb_lo;
    if (p.nblk_q <= 0) return cudaSuccess;
    p.sl2 = a.scale * 1.4426950408889634f;
    p.depth_packed = packed ? 1 : 0;
    p.depth_sel = a.depth_sel;
    p.kd_scale = a.kd_scale;
    p.vd_scale = a.vd_scale;
    p.status = a.status;
    p.wait_limit = a.wait_limit;
    const bool q8 = a.Ld > 0 && a.depth_q8;
    auto kern = q8 ? moda_fwd_tc_kernel<true> : moda_fwd_tc_kernel<false>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (err != cudaSuccess) return err;
    const long long grid = (long long)p.nblk_q * a.B * a.Hkv;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidValue;
    kern<<<(unsigned)grid, kThreads, kSmemBytes, s>>>(p);
    return cudaGetLastError();
}

}  // namespace moda
