// Tensor-core MoDA forward for sm_100a on CTA pairs: one tcgen05.mma with
// M = 256 drives the tensor cores of two SMs (cta_group::2).
//
// What it computes: the same as the single-CTA forward (moda_fwd_sm100.cu):
// "动态混合深度注意力机制MoDA技术解析" (mhpn.cn) §1.2, one softmax over
// [Q K_l^T || Q K_depth^T] / sqrt(d) times [V_l || V_depth]; §2.2, the online
// softmax state carried across key blocks and the dual mask.
//
// Why pairs were tried: in the single-CTA kernel the S = Q K^T MMAs read both
// operands from shared memory, 8 KB per 64-cycle K step (the SM's whole
// shared-memory operand bandwidth), and a clock64 timeline of one CTA at
// T = 16K showed them at ~100 cycles per 128x128x16 step. A pair MMA takes A
// from each CTA's own shared memory (its 128 query rows) and B half from each
// (N / 2): per SM 6 KB per K step for S, half of every K and V tile loaded by
// TMA, one issuing thread for both SMs.
// Measured result (B200): the S steps stay at ~100 cycles, and the item
// period grows from ~4370 to ~5120 cycles per SM (T = 16K: 3.19 ms against
// 2.13 ms): the period is set by each tile's softmax (~1750 cycles, MUFU-
// heavy) and its handoffs, which now span two SMs. So this kernel is a
// selectable variant (MODA_IMPL_TC2), not the default.
//
// Layout of the work:
//  * A cluster of two CTAs takes (b, kv-head, 4n tokens), n = 128 / G: CTA
//    rank r holds the query tiles of tokens [t0 + 2n r, t0 + 2n r + 2n) as two
//    128-row tiles (token-major GQA rows, as in the single-CTA kernel). MMA i
//    computes tile i of both CTAs at once.
//  * Key items: the causal sequence tiles up to the cluster's last token,
//    then the depth chunks of all 4n tokens' depth rows. Every tile takes
//    part in every item: the masks zero what a tile does not see (a sequence
//    tile past its tokens, another CTA's depth rows), so both CTAs' P are
//    valid for every pair MMA. This costs at most one causal item and half of
//    the depth items per CTA.
//  * B halves: K tiles split by keys (each CTA loads 64 of the 128 keys, all
//    features: N = keys for S = Q K^T), V tiles by features (each CTA loads 64
//    of the 128 features of all 128 keys: N = features for O = P V). Both TMA
//    loads of a slot complete on CTA 0's barrier (the 2-SM form of the copy,
//    never multicast); CTA 0's MMA thread waits there.
//  * Commits of the pair MMAs arrive on the barrier at the same offset in both
//    CTAs (s_full, empty, o_final, drain); each CTA's softmax publishes P to
//    CTA 0's p_full (cluster-scope arrivals, one per warp).
//  * Every wait is bounded; an expired wait sets the abort flag of both CTAs
//    and the device status word, and every thread still reaches the final
//    cluster barrier (no CTA exits while its peer may still touch its shared
//    memory or TMEM).
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

constexpr int kD = 128;
constexpr int kBN = 128;                       // keys per item
constexpr int kTileBytes = 128 * kD * 2;       // a 128-row bf16 tile: 32 KB
constexpr int kHalfBytes = kTileBytes / 2;     // one 64-column swizzled half
constexpr int kPart = kTileBytes / 2;          // this CTA's share of a K or V tile: 16 KB
constexpr int kStages = 8;                     // ring of 16 KB shares (K, V alternate)
constexpr int kThreads = 384;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kSoftmaxRegs = 216;
constexpr int kControlRegs = 72;
constexpr uint32_t kNoPollLimit = 0;
constexpr uint16_t kBoth = 0x3;                // CTA mask of the pair

struct PairFwdParams {
    CUtensorMap tm_q, tm_k, tm_v, tm_kd, tm_vd;  // k / kd boxes: 64 keys; v / vd boxes: 128 keys
    void* out;
    float* lse;
    int B, T, Hq, Hkv, G, n, Ld, nclu;  // nclu: clusters per (b, kv-head)
    float sl2;
    int depth_packed;
    const unsigned long long* depth_sel;
    unsigned int* status;
    unsigned int wait_limit;
};

struct __align__(8) PairBars {
    uint64_t q_full;            // CTA 0: both CTAs' Q tiles
    uint64_t full[kStages];     // CTA 0: both shares of a K or V tile
    uint64_t empty[kStages];    // both CTAs: the pair MMAs are done with a slot
    uint64_t s_full[2];         // both CTAs: S_i ready
    uint64_t p_full[2];         // CTA 0: P_i of both CTAs written (8 warp arrivals)
    uint64_t o_final[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};

constexpr int kSmemBytes = 2 * kTileBytes + kStages * kPart + 1024 /*bars*/ + 1024 /*align*/;
static_assert(kSmemBytes <= 232448, "shared memory per CTA");
static_assert(sizeof(PairBars) <= 1024, "barrier block");

__global__ void __launch_bounds__(kThreads, 1) moda_fwd_pair_kernel(const __grid_constant__ PairFwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;                           // 2 tiles
    uint8_t* sRing = smem + 2 * kTileBytes;       // kStages shares
    PairBars* bars = reinterpret_cast<PairBars*>(sRing + kStages * kPart);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const uint32_t rank = ptx::cluster_ctarank();
    const uint32_t wait_limit = p.wait_limit;
    volatile int* abort_flag = &bars->abort_flag;
    // the same barrier in CTA 0 (where the pair's TMA bytes and P arrivals go)
    auto lead_addr = [&](uint64_t* bar) { return ptx::mapa_shared(ptx::smem_u32(bar), 0); };
    auto flag_timeout = [&]() {
        *abort_flag = 1;
        ptx::st_cluster_u32(ptx::mapa_shared(ptx::smem_u32(&bars->abort_flag), rank ^ 1u), 1u);
        atomicOr(p.status, 1u);
    };

    // ---- work unit: (b, kv-head)-major, heaviest (latest) token blocks first
    const int c = blockIdx.x / 2;
    const int bh = c / p.nclu;
    const int cb = p.nclu - 1 - c % p.nclu;
    const int b = bh / p.Hkv, kvh = bh % p.Hkv;
    const int n = p.n;
    const int tc0 = cb * 4 * n;                    // the cluster's first token
    const int t0 = tc0 + (int)rank * 2 * n;        // this CTA's first token
    const int last = min(p.T - 1, tc0 + 4 * n - 1);
    const int n_seq = last / kBN + 1;
    const int ntok = last - tc0 + 1;               // the cluster's tokens inside the sequence
    const int n_dep = (ntok * p.Ld + kBN - 1) / kBN;
    const int n_items = n_seq + n_dep;

    if (threadIdx.x == 0) {
        ptx::mbar_init(&bars->q_full, 1);
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(&bars->full[s], 1);
            ptx::mbar_init(&bars->empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&bars->s_full[i], 1);
            ptx::mbar_init(&bars->p_full[i], 8);  // four warps in each CTA
            ptx::mbar_init(&bars->o_final[i], 1);
        }
        ptx::mbar_init(&bars->drain, 1);
        bars->abort_flag = 0;
        ptx::fence_barrier_init();
        ptx::fence_proxy_async_smem();
    }
    if (warp == 0) {
        ptx::tmem_alloc_pair(&bars->tmem_base, 512);
        ptx::tmem_relinquish_pair();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();  // both CTAs' barriers exist before any remote arrival
    ptx::tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp >= 8) ptx::setmaxnreg_dec<kControlRegs>();
    if (warp == kProducerWarp) {
        // The whole warp runs the schedule; lane 0 issues the copies.
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
        if (rank == 0) ptx::mbar_arrive_expect_tx_lead(&bars->q_full, 2 * 2 * kTileBytes, lead);
        for (int i = 0; i < 2; ++i)
            for (int hf = 0; hf < 2; ++hf)
                ptx::tma_load_4d_pair_lead(sQ + i * kTileBytes + hf * kHalfBytes, &p.tm_q, lead_addr(&bars->q_full),
                                           hf * 64, kvh * p.G, t0 + i * n, b, lead);
        const uint32_t full0 = lead_addr(&bars->full[0]);  // CTA 0's full[0]; full[s] is 8 s bytes on
        int seq = 0;
        bool ok = true;
        for (int x = 0; x < n_items && ok; ++x) {
            for (int kv = 0; kv < 2; ++kv, ++seq) {
                const int st = seq % kStages;
                const uint32_t ph = (seq / kStages) & 1;
                if (!__all_sync(0xffffffffu, ptx::mbar_wait(&bars->empty[st], ph ^ 1, wait_limit, abort_flag))) {
                    if (lead) flag_timeout();
                    ok = false;
                    break;
                }
                if (rank == 0) ptx::mbar_arrive_expect_tx_lead(&bars->full[st], 2 * kPart, lead);
                uint8_t* dst = sRing + st * kPart;
                const uint32_t fb = full0 + 8u * (uint32_t)st;
                if (kv == 0) {
                    // K: keys [row0 + 64 rank, +64), both 64-feature halves
                    const int row0 = (x < n_seq ? x * kBN : tc0 * p.Ld + (x - n_seq) * kBN) + 64 * (int)rank;
                    const CUtensorMap* m = x < n_seq ? &p.tm_k : &p.tm_kd;
                    for (int hf = 0; hf < 2; ++hf) {
                        if (x >= n_seq && p.depth_packed)
                            ptx::tma_load_4d_pair_lead(dst + hf * (kPart / 2), m, fb, hf * 64, row0, kvh, b, lead);
                        else
                            ptx::tma_load_4d_pair_lead(dst + hf * (kPart / 2), m, fb, hf * 64, kvh, row0, b, lead);
                    }
                } else {
                    // V: features [64 rank, +64) of all 128 keys
                    const int row0 = x < n_seq ? x * kBN : tc0 * p.Ld + (x - n_seq) * kBN;
                    const CUtensorMap* m = x < n_seq ? &p.tm_v : &p.tm_vd;
                    if (x >= n_seq && p.depth_packed)
                        ptx::tma_load_4d_pair_lead(dst, m, fb, 64 * (int)rank, row0, kvh, b, lead);
                    else
                        ptx::tma_load_4d_pair_lead(dst, m, fb, 64 * (int)rank, kvh, row0, b, lead);
                }
            }
        }
        // Drain (CTA 0, where every load of the pair completes): all loads
        // land before the pair can exit.
        if (rank == 0) {
            ptx::mbar_wait(&bars->q_full, 0, kNoPollLimit, nullptr);
            for (int s = (seq > kStages ? seq - kStages : 0); s < seq; ++s)
                ptx::mbar_wait(&bars->full[s % kStages], (s / kStages) & 1, kNoPollLimit, nullptr);
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        if (rank == 0 && lane == 0) {
            // One thread of CTA 0 issues every pair MMA and commit.
            constexpr uint32_t idesc_qk = ptx::idesc_bf16_f32(256, kBN, 0, 0);
            constexpr uint32_t idesc_pv = ptx::idesc_bf16_f32(256, kD, 0, 1);
            const uint32_t sQa = ptx::smem_u32(sQ);
            const uint32_t sRa = ptx::smem_u32(sRing);
            const uint64_t dq0 = ptx::umma_desc_sw128(sQa, 16, 1024);
            const uint64_t dq1 = ptx::umma_desc_sw128(sQa + kTileBytes, 16, 1024);
            auto wait = [&](uint64_t* bar, uint32_t parity) { return ptx::mbar_wait(bar, parity, wait_limit, abort_flag); };
            bool ok = wait(&bars->q_full, 0);
            ptx::tc_fence_after();
            // S_i = Q_i K^T for the K share in ring slot `SEQ` (K step k: 32 B
            // within the 128-byte row, 16 KB / 8 KB per 64-feature half of the
            // Q tile / the 64-key K share)
            auto issue_s = [&](int i, int sq) {
                const uint64_t kd_ = ptx::umma_desc_sw128(sRa + (sq % kStages) * kPart, 16, 1024);
#pragma unroll
                for (int k = 0; k < kD / 16; ++k) {
                    const uint64_t qo = (uint64_t)((k >> 2) * (kHalfBytes >> 4) + (k & 3) * 2);
                    const uint64_t ko = (uint64_t)((k >> 2) * ((kPart / 2) >> 4) + (k & 3) * 2);
                    ptx::mma_ss_pair(tmem + i * 128, (i ? dq1 : dq0) + qo, kd_ + ko, idesc_qk, k > 0);
                }
                ptx::mma_commit_pair(&bars->s_full[i], kBoth);
            };
            if (ok) ok = wait(&bars->full[0], 0);
            ptx::tc_fence_after();
            if (ok) {
                issue_s(0, 0);
                issue_s(1, 0);
                ptx::mma_commit_pair(&bars->empty[0], kBoth);
            }
            for (int x = 0; x < n_items && ok; ++x) {
                const int sv = 2 * x + 1, sk = 2 * x + 2;
                const bool next = x + 1 < n_items;
                if (!(ok = wait(&bars->full[sv % kStages], (sv / kStages) & 1))) break;
                ptx::tc_fence_after();
                // V share: 128 keys x 64 features, MN-major (16 keys = 2 KB per K step)
                const uint64_t vd = ptx::umma_desc_sw128(sRa + (sv % kStages) * kPart, kHalfBytes, 1024);
                bool k_ready = false;
#pragma unroll 1
                for (int i = 0; i < 2; ++i) {
                    // O_i += P_i V once both CTAs have published P_i
                    if (!ptx::mbar_wait_cluster(&bars->p_full[i], x & 1, wait_limit, abort_flag)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        ptx::mma_ts_pair(tmem + 256 + i * 128, tmem + i * 128 + k * 8, vd + (uint64_t)(k * 128),
                                         idesc_pv, (x > 0 || k > 0) ? 1u : 0u);
                    if (next) {
                        if (!k_ready) {
                            if (!(ok = wait(&bars->full[sk % kStages], (sk / kStages) & 1))) break;
                            ptx::tc_fence_after();
                            k_ready = true;
                        }
                        issue_s(i, sk);
                    }
                }
                if (!ok) break;
                ptx::mma_commit_pair(&bars->empty[sv % kStages], kBoth);
                if (next) ptx::mma_commit_pair(&bars->empty[sk % kStages], kBoth);
            }
            if (!ok) flag_timeout();
            if (ok) {
                ptx::mma_commit_pair(&bars->o_final[0], kBoth);
                ptx::mma_commit_pair(&bars->o_final[1], kBoth);
            }
            // Drain: every pair MMA completes before either CTA frees TMEM.
            ptx::mma_commit_pair(&bars->drain, kBoth);
        }
        // both CTAs: the pair's MMAs (which touch this CTA's shared memory
        // and TMEM) are done
        if (lane == 0) ptx::mbar_wait(&bars->drain, 0, kNoPollLimit, nullptr);
        __syncwarp();
    } else if (warp < 8) {
        // ------------------------------------------------ softmax warpgroups
        ptx::setmaxnreg_inc<kSoftmaxRegs>();
        const int i = warp / 4;            // query tile
        const int r = (warp % 4) * 32 + lane;  // row = TMEM lane
        const uint32_t lane_off = (uint32_t)((warp % 4) * 32) << 16;
        const uint32_t tS = tmem + lane_off + i * 128;
        const uint32_t tO = tmem + lane_off + 256 + i * 128;
        const int tlc = (int)rank * 2 * n + i * n + r / p.G;  // token offset in the cluster
        const int t = tc0 + tlc;
        const int h = kvh * p.G + r % p.G;
        const float sl2 = p.sl2;
        const bool has_sel = p.depth_sel != nullptr;
        const unsigned long long sel =
            has_sel && t < p.T ? p.depth_sel[(long long)b * p.T + t] & depth_slot_bits(p.Ld) : 0ull;
        const uint32_t pfull_lead = lead_addr(&bars->p_full[i]);
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        for (int x = 0; x < n_items; ++x) {
            const bool got = ptx::mbar_wait(&bars->s_full[i], x & 1, wait_limit, abort_flag);
            if (!__all_sync(0xffffffffu, got)) {
                flag_timeout();
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            softmax_item(tS, tO, x < n_seq, x * kBN, t, tlc * p.Ld - (x - n_seq) * kBN, p.Ld, has_sel, sel, sl2, x,
                         m, l);
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive_cluster(pfull_lead);
        }
        if (ok) {
            const bool got = ptx::mbar_wait(&bars->o_final[i], 0, wait_limit, abort_flag);
            if (!__all_sync(0xffffffffu, got)) {
                flag_timeout();
                ok = false;
            }
        }
        ptx::tc_fence_after();
        if (ok) {
            const bool valid = t < p.T;
            const float inv = 1.f / l;
            __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.out) + (((long long)b * p.T + (valid ? t : 0)) * p.Hq + h) * kD;
#pragma unroll 1
            for (int cc = 0; cc < 4; ++cc) {
                uint32_t o[32];
                ptx::tmem_ld32(tO + cc * 32, o);
                ptx::tmem_wait_ld();
                uint32_t w[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    w[e] = ptx::pack_bf16x2(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
                if (valid) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + cc * 32);
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
    ptx::cluster_sync();  // neither CTA leaves while its peer may still signal it
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc_pair(tmem, 512);
    }
}

}  // namespace

bool fwd_pair_supported(const FwdArgs& a) {
    // the single-CTA kernel's conditions; 8-bit depth stays on that kernel
    return fwd_tc_supported(a) && !a.depth_q8;
}

cudaError_t launch_fwd_pair(const FwdArgs& a, cudaStream_t s) {
    PairFwdParams p;
    memset(&p, 0, sizeof(p));
    const int G = a.G, n = 128 / G;
    const cuuint64_t e = 2;
    {
        const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)a.Hq, (cuuint64_t)a.T, (cuuint64_t)a.B};
        const cuuint64_t st[3] = {kD * e, (cuuint64_t)a.Hq * kD * e, (cuuint64_t)a.T * a.Hq * kD * e};
        const cuuint32_t box[4] = {64, (cuuint32_t)G, (cuuint32_t)n, 1};
        if (!make_tmap_bf16_4d(&p.tm_q, a.q, dims, st, box)) return cudaErrorInvalidValue;
    }
    {
        const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)a.Hkv, (cuuint64_t)a.T, (cuuint64_t)a.B};
        const cuuint64_t st[3] = {kD * e, (cuuint64_t)a.Hkv * kD * e, (cuuint64_t)a.T * a.Hkv * kD * e};
        const cuuint32_t kbox[4] = {64, 1, 64, 1}, vbox[4] = {64, 1, (cuuint32_t)kBN, 1};
        if (!make_tmap_bf16_4d(&p.tm_k, a.k, dims, st, kbox)) return cudaErrorInvalidValue;
        if (!make_tmap_bf16_4d(&p.tm_v, a.v, dims, st, vbox)) return cudaErrorInvalidValue;
    }
    const bool packed = a.Ld > 0 && a.sdep.si == kD;  // [B, Hkv, T*Ld, d]
    if (a.Ld > 0) {
        const cuuint64_t rows = (cuuint64_t)a.T * a.Ld;
        if (packed) {
            const cuuint64_t dims[4] = {(cuuint64_t)kD, rows, (cuuint64_t)a.Hkv, (cuuint64_t)a.B};
            const cuuint64_t st[3] = {kD * e, rows * kD * e, (cuuint64_t)a.Hkv * rows * kD * e};
            const cuuint32_t kbox[4] = {64, 64, 1, 1}, vbox[4] = {64, (cuuint32_t)kBN, 1, 1};
            if (!make_tmap_bf16_4d(&p.tm_kd, a.kd, dims, st, kbox)) return cudaErrorInvalidValue;
            if (!make_tmap_bf16_4d(&p.tm_vd, a.vd, dims, st, vbox)) return cudaErrorInvalidValue;
        } else {
            const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)a.Hkv, rows, (cuuint64_t)a.B};
            const cuuint64_t st[3] = {kD * e, (cuuint64_t)a.Hkv * kD * e, rows * a.Hkv * kD * e};
            const cuuint32_t kbox[4] = {64, 1, 64, 1}, vbox[4] = {64, 1, (cuuint32_t)kBN, 1};
            if (!make_tmap_bf16_4d(&p.tm_kd, a.kd, dims, st, kbox)) return cudaErrorInvalidValue;
            if (!make_tmap_bf16_4d(&p.tm_vd, a.vd, dims, st, vbox)) return cudaErrorInvalidValue;
        }
    } else {
        p.tm_kd = p.tm_k;
        p.tm_vd = p.tm_v;
    }
    p.out = a.out;
    p.lse = a.lse;
    p.B = a.B; p.T = a.T; p.Hq = a.Hq; p.Hkv = a.Hkv; p.G = G; p.n = n; p.Ld = a.Ld;
    p.nclu = (a.T + 4 * n - 1) / (4 * n);
    p.sl2 = a.scale * 1.4426950408889634f;
    p.depth_packed = packed ? 1 : 0;
    p.depth_sel = a.depth_sel;
    p.status = a.status;
    p.wait_limit = a.wait_limit;
    cudaError_t err = cudaFuncSetAttribute(moda_fwd_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (err != cudaSuccess) return err;
    const long long clusters = (long long)p.nclu * a.B * a.Hkv;
    if (2 * clusters > 0x7fffffffLL) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * clusters), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, moda_fwd_pair_kernel, p);
}

}  // namespace moda
