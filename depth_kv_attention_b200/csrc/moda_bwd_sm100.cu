// Tensor-core MoDA backward for sm_100a (bf16, d = 128, 128 % G == 0).
//
// The pages give no backward pass; this computes the derivative of the MoDA
// forward ("动态混合深度注意力机制MoDA技术解析" (mhpn.cn) §1.2 formula, §2.2 dual
// mask) with the usual softmax-Jacobian identities:
//   P = exp(s - lse),  dP = dout . v,  D = sum_j P_j dP_j,  dS = P * (dP - D)
//   dq = scale (sum_j dS_j k_j + sum_i dS'_i kd_i)
//   dk_j = scale sum dS_j q,  dv_j = sum P_j dout   (rows t >= j, G heads)
//   dkd_i = scale sum_h dS'_i q,  dvd_i = sum_h P'_i dout   (same token)
//
// Launch sequence (one stream):
//   1. dq: query-major tensor-core kernel over the causal key tiles and the
//      query tile's own depth chunks. It forms the estimate D~ = <dout, out>
//      from the stored output, sees all keys of its rows, and so also forms
//      the exact D = D~ + sum_j P_j (dP_j - D~) and corrects dq for D - D~;
//      dq accumulates in TMEM and is written once, in bf16
//   2. one launch of the KV-major tensor-core kernel (reads the exact D):
//      dk, dv CTAs first (partial sums of a key tile over a chunk of query
//      tiles go to fp32 accumulators with vector reductions), then dkd, dvd
//      CTAs (128-row depth chunks as the key tiles, a same-token mask, each
//      depth row owned by one CTA, bf16 stores), which fill the SMs the
//      last wave of dk, dv CTAs leaves idle
//   3. dk, dv = bf16(accumulators)
// Splitting dq from dk/dv recomputes S and dP once more but removes the
// per-pair fp32 dq reductions, which for wide GQA (G = 32, 4 tokens per
// 128-row tile) would move gigabytes through L2.
//
// Both kernels put query rows in the forward's token-major GQA order (a
// 128-row tile = n = 128/G tokens x G heads). Warp 8 issues the TMA loads
// (the whole warp runs the schedule, lane 0 issues), lane 0 of warp 9 issues
// every tcgen05.mma and commit, and warps 0-7 (two warpgroups, one per
// 64-column half of every TMEM tile) do the elementwise work, one thread per
// TMEM lane.
#include <cuda_bf16.h>

#include <cmath>
#include <cstring>
#include <type_traits>

#include "depth_mask.cuh"
#include "moda_internal.h"
#include "sm100_ptx.cuh"
#include "tmap_host.h"

namespace moda {
namespace {

constexpr int kD = 128;
constexpr int kBK = 128;          // keys per key tile
constexpr int kTile = 128 * kD * 2;
constexpr int kHalf = kTile / 2;
// Warps 0-7 compute (two warpgroups: column halves 0-63 and 64-127 of every
// TMEM tile; warp w reaches TMEM lanes 32*(w%4) ..), 8 TMA producer, 9 MMA.
constexpr int kThreads = 320;
constexpr int kComputeThreads = 256;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr float kLog2e = 1.4426950408889634f;
// Of every 8 column pairs, pairs kBwdPolyFrom..7 take exp2 from the FMA-pipe
// polynomial, the rest from MUFU (in these kernels the exponentials sit on
// the critical path of one compute warp per SM sub-partition).
#ifndef MODA_BWD_POLY_FROM
#define MODA_BWD_POLY_FROM 8
#endif
constexpr int kBwdPolyFrom = MODA_BWD_POLY_FROM;
__device__ __forceinline__ float2 exp2_pair(float2 x, int pair) {
    if ((pair & 7) >= kBwdPolyFrom) return ptx::exp2_poly2(x);
    return make_float2(ptx::ex2(x.x), ptx::ex2(x.y));
}

__device__ __forceinline__ uint64_t kdesc(uint32_t tile) { return ptx::umma_desc_sw128(tile, 16, 1024); }
__device__ __forceinline__ uint64_t mndesc(uint32_t tile) { return ptx::umma_desc_sw128(tile, kHalf, 1024); }
// K step k of a K-major tile: 32 B within the 128-byte row, 16 KB per half.
__device__ __forceinline__ uint64_t koff(int k) { return (uint64_t)((k >> 2) * (kHalf >> 4) + (k & 3) * 2); }
// K step k of an MN-major tile: 16 rows of 128 B.
__device__ __forceinline__ uint64_t mnoff(int k) { return (uint64_t)(k * 128); }

__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}
// Barrier 1 + hs spans the 128 compute threads of column half hs only.
__device__ __forceinline__ void half_sync(int hs) {
    asm volatile("bar.sync %0, 128;" ::"r"(1 + hs) : "memory");
}
// AND of `v` over the 128 compute threads of column half hs (a barrier too):
// every warp of the half takes the same branch after a bounded wait, so none
// is left waiting at a later named barrier.
__device__ __forceinline__ bool half_all(int hs, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.and.pred po, %2, 128, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(1 + hs)
        : "memory");
    return r != 0;
}
// TMEM column of K step k (16 rows of the reduced dimension = 8 packed
// columns) of a bf16 A operand whose two column halves each wrote their
// packed values at the start of their own 64 columns.
__device__ __forceinline__ uint32_t acol(int k) { return (uint32_t)((k >> 2) * 64 + (k & 3) * 8); }

struct __align__(8) Bars {
    uint64_t kv_full;            // dk/dv kernel: K, V tile | dq kernel: Q, dO tile
    uint64_t full[4];            // ring slots
    uint64_t empty[4];
    uint64_t s_full, dp_full, p_full, p_full2, fin, drain, dp_read;
    uint64_t p_ready;            // dq kernel: P of the item written (one arrival per compute warp)
    uint32_t tmem_base;
    int abort_flag;
};

__device__ __forceinline__ void flag_timeout(unsigned int* status, Bars* bars) {
    *reinterpret_cast<volatile int*>(&bars->abort_flag) = 1;
    atomicOr(status, 1u);
}

// p_count: arrivals that publish P, one per compute warp (the dQ kernel: 8 on
// p_full; the dK/dV kernel: each 4-warp half on its own p_full / p_full2).
// Per-thread arrivals on one barrier word would serialise on the chain.
__device__ __forceinline__ void init_bars(Bars* bars, int stages, int p_count) {
    ptx::mbar_init(&bars->kv_full, 1);
    for (int s = 0; s < stages; ++s) {
        ptx::mbar_init(&bars->full[s], 1);
        ptx::mbar_init(&bars->empty[s], 1);
    }
    ptx::mbar_init(&bars->s_full, 1);
    ptx::mbar_init(&bars->dp_full, 1);
    ptx::mbar_init(&bars->p_full, p_count);
    ptx::mbar_init(&bars->p_full2, p_count);
    ptx::mbar_init(&bars->fin, 1);
    ptx::mbar_init(&bars->drain, 1);
    ptx::mbar_init(&bars->dp_read, 8);
    ptx::mbar_init(&bars->p_ready, 8);
    bars->abort_flag = 0;
    ptx::fence_barrier_init();
    ptx::fence_proxy_async_smem();
}

// ===================================================================== dk, dv
struct DkvParams {
    CUtensorMap tm_q, tm_do, tm_k, tm_v, tm_kd, tm_vd;
    const float* lse;
    const float* rowD;
    float* dk_acc;  // sequence mode: [B,T,Hkv,d] fp32, zeroed before the launch
    float* dv_acc;
    void* dkd;      // depth mode: [B,T,Ld,Hkv,d] bf16 outputs
    void* dvd;
    int Ld;
    const unsigned long long* depth_sel;  // depth mode: [B,T] slot masks or null
    int B, T, Hq, Hkv, G, n, gshift, qchunk;
    // grid: n_seq_ctas sequence-mode CTAs (key tile fastest, then chunk of
    // query tokens, then (b, kv-head)), then n_dep_chunks depth-mode CTAs per
    // (b, kv-head) (depth chunk fastest)
    int nkt, n_chunks, n_dep_chunks;
    long long n_seq_ctas;
    float sl2, scale;
    unsigned int* status;
    unsigned int wait_limit;
};
constexpr int kDkvStages = 2;  // ring of (Q, dO) pairs
constexpr int kDkvSmem = 2 * kTile + kDkvStages * 2 * kTile + 2 * 128 * 4 + 256 + 1024;
static_assert(kDkvSmem <= 232448, "shared memory per CTA");
static_assert(sizeof(Bars) <= 256, "barrier block");

// One launch holds both kinds of CTA: the sequence-mode CTAs first, then the
// depth-mode ones, which are short and fill the SMs that the last wave of
// long sequence-mode CTAs leaves idle.
// Sequence mode: one CTA per (key tile, chunk of query tokens, (b, kv-head)),
// causal mask, partial sums reduced into fp32 accumulators.
// Depth mode (the depth keys' gradients dkd, dvd): the "key tile" is a
// 128-row depth chunk of the [B, T*Ld, Hkv, d] view, the query tiles are
// those holding the chunk's tokens, the mask keeps each depth row to its own
// token's G heads, and since one CTA owns every row of its chunk the results
// are written directly in bf16.
// Each 128-row query tile is processed as two halves of 64 query rows that
// ping-pong like the forward's two query tiles: while the compute warps of
// one half form P^T and dS^T, the tensor core runs the other half's MMAs.
// TMEM: [S^T | dP^T] of half 0, [S^T | dP^T] of half 1 (64 columns each),
// then dV | dK (128 columns each).
// Per half h of query tile i: S^T_h = K Q_h^T and dP^T_h = V dO_h^T
// (N = 64); the 128 compute threads of half h (thread = key) write P^T_h and
// dS^T_h in bf16 over them; dV += P^T_h dO_h and dK += dS^T_h Q_h take them
// as TMEM A operands (K = 64 queries). MMA issue order per tile:
// PV_0(i), S/dP_0(i+1), PV_1(i), S/dP_1(i+1), so a half's next S^T / dP^T
// overwrite its P^T / dS^T only after they are read.
__global__ void __launch_bounds__(kThreads, 1) moda_bwd_dkdv_kernel(const __grid_constant__ DkvParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sK = smem;
    uint8_t* sV = smem + kTile;
    uint8_t* sRing = smem + 2 * kTile;  // stage s: Q at +2s*kTile, dO at +(2s+1)*kTile
    float* sStat = reinterpret_cast<float*>(sRing + kDkvStages * 2 * kTile);  // [-lse2 | -D] of the query tile
    Bars* bars = reinterpret_cast<Bars*>(sStat + 256);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    volatile int* abort_flag = &bars->abort_flag;
    // (key tile or depth chunk, chunk of query tokens, (b, kv-head)) of this CTA
    const bool depth_mode = (long long)blockIdx.x >= p.n_seq_ctas;
    int bx, by, bz;
    if (!depth_mode) {
        const int r = (int)blockIdx.x / p.nkt;
        bx = (int)blockIdx.x % p.nkt;
        by = r % p.n_chunks;
        bz = r / p.n_chunks;
    } else {
        const long long r = (long long)blockIdx.x - p.n_seq_ctas;
        bx = (int)(r % p.n_dep_chunks);
        by = 0;
        bz = (int)(r / p.n_dep_chunks);
    }
    const CUtensorMap* tm_kx = depth_mode ? &p.tm_kd : &p.tm_k;
    const CUtensorMap* tm_vx = depth_mode ? &p.tm_vd : &p.tm_v;
    const int b = bz / p.Hkv, kvh = bz % p.Hkv;
    const int j0 = bx * kBK;  // first key row (sequence) or depth row (depth mode)
    const int n = p.n;
    int t_first, nq;
    if (depth_mode) {
        // tokens whose depth rows meet [j0, j0 + 128), whole query tiles
        const int last_row = min(j0 + kBK, p.T * p.Ld) - 1;
        t_first = (j0 / p.Ld) / n * n;
        nq = (last_row / p.Ld - t_first) / n + 1;
    } else {
        // A chunk is qchunk query tiles of absolute tokens [c*qchunk*n, ...);
        // the CTAs in flight at once cover one or two chunks. Key tiles that
        // no row of the chunk can see exit at once.
        const int c_lo = by * p.qchunk * n;
        const int c_hi = min(p.T, (by + 1) * p.qchunk * n);
        t_first = max(j0, c_lo);  // a multiple of n
        if (t_first >= c_hi) return;
        nq = (c_hi - t_first + n - 1) / n;
    }

    if (threadIdx.x == 0) init_bars(bars, kDkvStages, kComputeThreads / 64);
    if (warp == 0) {
        ptx::tmem_alloc(&bars->tmem_base, 512);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
        return __all_sync(0xffffffffu, ptx::mbar_wait(bar, parity, p.wait_limit, abort_flag));
    };
    auto wait_one = [&](uint64_t* bar, uint32_t parity) {
        return ptx::mbar_wait(bar, parity, p.wait_limit, abort_flag);
    };

    if (warp == kProducerWarp) {
        const uint32_t lead = lane == 0;
        if (lead) {
            ptx::prefetch_tmap(&p.tm_q);
            ptx::prefetch_tmap(&p.tm_do);
            ptx::prefetch_tmap(tm_kx);
            ptx::prefetch_tmap(tm_vx);
        }
        ptx::mbar_arrive_expect_tx_lead(&bars->kv_full, 2 * kTile, lead);
        for (int hf = 0; hf < 2; ++hf) {
            ptx::tma_load_4d_lead(sK + hf * kHalf, tm_kx, &bars->kv_full, hf * 64, kvh, j0, b, lead);
            ptx::tma_load_4d_lead(sV + hf * kHalf, tm_vx, &bars->kv_full, hf * 64, kvh, j0, b, lead);
        }
        int issued = 0;
        for (int i = 0; i < nq; ++i) {
            const int st = i % kDkvStages;
            if (!wait_all(&bars->empty[st], ((i / kDkvStages) & 1) ^ 1)) {
                if (lead) flag_timeout(p.status, bars);
                break;
            }
            ptx::mbar_arrive_expect_tx_lead(&bars->full[st], 2 * kTile, lead);
            const int tq0 = t_first + i * n;
            for (int hf = 0; hf < 2; ++hf) {
                ptx::tma_load_4d_lead(sRing + (2 * st) * kTile + hf * kHalf, &p.tm_q, &bars->full[st], hf * 64,
                                      kvh * p.G, tq0, b, lead);
                ptx::tma_load_4d_lead(sRing + (2 * st + 1) * kTile + hf * kHalf, &p.tm_do, &bars->full[st],
                                      hf * 64, kvh * p.G, tq0, b, lead);
            }
            issued = i + 1;
        }
        ptx::mbar_wait(&bars->kv_full, 0, 0, nullptr);
        for (int i = (issued > kDkvStages ? issued - kDkvStages : 0); i < issued; ++i)
            ptx::mbar_wait(&bars->full[i % kDkvStages], (i / kDkvStages) & 1, 0, nullptr);
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // One thread runs the MMA schedule (a single-thread tcgen05.mma issue
        // costs about 60 cycles, a warp-wide one predicated on one lane 80-90,
        // against 64 cycles of tensor work for a 128x128x16 MMA; measured on
        // the B200).
        if (lane == 0) {
            constexpr uint32_t idesc_half = ptx::idesc_bf16_f32(128, 64, 0, 0);
            constexpr uint32_t idesc_ts = ptx::idesc_bf16_f32(128, kD, 0, 1);
            const uint64_t dK = kdesc(ptx::smem_u32(sK)), dV = kdesc(ptx::smem_u32(sV));
            const uint32_t aRing = ptx::smem_u32(sRing);
            uint64_t* s_ready[2] = {&bars->s_full, &bars->dp_full};
            uint64_t* p_ready[2] = {&bars->p_full, &bars->p_full2};
            // S^T_h = K Q_h^T and dP^T_h = V dO_h^T for query half h of the
            // tile in ring stage st (rows 64h.. of each 64-column half of the
            // K-major Q / dO tile: 64 rows of 128 B = 512 descriptor units)
            auto issue_sdp = [&](int st, int h) {
                const uint32_t aQ = aRing + (2 * st) * kTile, aDO = aRing + (2 * st + 1) * kTile;
                const uint64_t rows = (uint64_t)(h * 512);
                const uint64_t dQk = kdesc(aQ) + rows, dOk = kdesc(aDO) + rows;
#pragma unroll
                for (int k = 0; k < kD / 16; ++k)
                    ptx::mma_ss(tmem + 128 * h, dK + koff(k), dQk + koff(k), idesc_half, k > 0);
#pragma unroll
                for (int k = 0; k < kD / 16; ++k)
                    ptx::mma_ss(tmem + 128 * h + 64, dV + koff(k), dOk + koff(k), idesc_half, k > 0);
                ptx::mma_commit(s_ready[h]);
            };
            // dV += P^T_h dO_h and dK += dS^T_h Q_h: K steps 4h .. 4h+3 of the
            // MN-major dO / Q tile, A operands from half h's TMEM columns
            auto issue_pv = [&](int st, int h, bool first) {
                const uint32_t aQ = aRing + (2 * st) * kTile, aDO = aRing + (2 * st + 1) * kTile;
                const uint64_t dQm = mndesc(aQ), dOm = mndesc(aDO);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    ptx::mma_ts(tmem + 256, tmem + 128 * h + 8 * kk, dOm + mnoff(4 * h + kk), idesc_ts,
                                (first && kk == 0) ? 0u : 1u);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    ptx::mma_ts(tmem + 384, tmem + 128 * h + 64 + 8 * kk, dQm + mnoff(4 * h + kk), idesc_ts,
                                (first && kk == 0) ? 0u : 1u);
            };
            bool ok = wait_one(&bars->kv_full, 0) && wait_one(&bars->full[0], 0);
            if (!ok) flag_timeout(p.status, bars);
            ptx::tc_fence_after();
            if (ok) {
                issue_sdp(0, 0);
                issue_sdp(0, 1);
            }
            for (int i = 0; i < nq && ok; ++i) {
                const int st = i % kDkvStages, st2 = (i + 1) % kDkvStages;
                const bool next = i + 1 < nq;
                for (int h = 0; h < 2; ++h) {
                    if (!wait_one(p_ready[h], i & 1)) {
                        flag_timeout(p.status, bars);
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    issue_pv(st, h, i == 0 && h == 0);
                    if (h == 1) ptx::mma_commit(&bars->empty[st]);  // Q, dO of tile i are read
                    if (next) {
                        if (h == 0) {
                            if (!wait_one(&bars->full[st2], ((i + 1) / kDkvStages) & 1)) {
                                flag_timeout(p.status, bars);
                                ok = false;
                                break;
                            }
                            ptx::tc_fence_after();
                        }
                        issue_sdp(st2, h);
                    }
                }
            }
            if (ok) ptx::mma_commit(&bars->fin);
            ptx::mma_commit(&bars->drain);
            ptx::mbar_wait(&bars->drain, 0, 0, nullptr);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ compute warps
        // Half hs: query rows 64hs .. 64hs+63 of every tile (its own S^T /
        // dP^T columns 128hs ..), and feature columns 64hs .. of dV / dK in
        // the epilogue.
        const int hs = warp / 4;
        const int r = (warp % 4) * 32 + lane;  // TMEM lane
        const uint32_t lane_off = (uint32_t)((warp % 4) * 32) << 16;
        const int j = j0 + r;            // this thread's key
        // depth mode: is depth row j (slot j % Ld of token j / Ld) selected?
        const bool j_selected = !depth_mode || !p.depth_sel || j >= p.T * p.Ld ||
                                ((p.depth_sel[(long long)b * p.T + j / p.Ld] >> (j % p.Ld)) & 1ull);
        const float sl2 = p.sl2;
        const int gshift = p.gshift;
        bool ok = true;
        // lse (log2 units) and D of query row 64hs + r (r < 64) of query tile
        // i, loaded one tile ahead so the global-memory latency stays off the
        // critical path.
        auto load_stat = [&](int i, float& l2, float& dd) {
            const int rr = 64 * hs + r;
            const int t = t_first + i * n + (rr >> gshift), h = kvh * p.G + (rr & (p.G - 1));
            if (t < p.T) {
                const long long ix = ((long long)b * p.Hq + h) * p.T + t;
                l2 = p.lse[ix] * kLog2e;
                dd = p.rowD[ix];
            } else {
                l2 = INFINITY;  // rows past T: P = 0
                dd = 0.f;
            }
        };
        float nl2 = INFINITY, nD = 0.f;
        if (r < 64) load_stat(0, nl2, nD);
        for (int i = 0; i < nq; ++i) {
            const int tq0 = t_first + i * n;
            float* st_lse = sStat;
            float* st_D = sStat + 128;
            half_sync(hs);  // this half's readers of the previous tile are done
            if (r < 64) {
                st_lse[64 * hs + r] = -nl2;  // stored negated: the packed FMA / ADD below add them
                st_D[64 * hs + r] = -nD;
                if (i + 1 < nq) load_stat(i + 1, nl2, nD);
            }
            const bool got = ptx::mbar_wait(hs ? &bars->dp_full : &bars->s_full, i & 1, p.wait_limit, abort_flag);
            if (!half_all(hs, got)) {  // also publishes this half's st_lse / st_D
                flag_timeout(p.status, bars);
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            // Visible rows rr form a range [lo_r, hi_r): sequence mode, key j
            // is seen by rows of tokens tq0 + (rr >> gshift) >= j; depth mode,
            // depth row j is seen only by the rows of its own token j / Ld.
            int lo_r, hi_r;
            if (depth_mode) {
                const int td = j < p.T * p.Ld ? j / p.Ld : -1;
                lo_r = (td - tq0) * p.G;
                hi_r = (td < 0 || !j_selected) ? lo_r : lo_r + p.G;
            } else {
                lo_r = j > tq0 ? (j - tq0) << gshift : 0;
                hi_r = 128;
            }
            const uint32_t tH = tmem + lane_off + 128 * hs;  // this half's S^T | dP^T
            // every query row of this half visible to every key of the warp:
            // the loop without the per-element range test (warp-uniform)
            const bool all_vis = __all_sync(0xffffffffu, lo_r <= 64 * hs && hi_r >= 64 * hs + 64);
            auto tile = [&](auto masked) {
#pragma unroll 1
                for (int c = 0; c < 2; ++c) {
                    uint32_t sr[32], dr[32];
                    ptx::tmem_ld32(tH + 32 * c, sr);
                    ptx::tmem_ld32(tH + 64 + 32 * c, dr);
                    ptx::tmem_wait_ld();
                    uint32_t pp[16], dd[16];
#pragma unroll
                    for (int e2 = 0; e2 < 16; ++e2) {
                        const int r0 = 64 * hs + 32 * c + 2 * e2;  // query row of the tile
                        const float2 nl = *reinterpret_cast<const float2*>(st_lse + r0);
                        const float2 nd = *reinterpret_cast<const float2*>(st_D + r0);
                        float2 pv = exp2_pair(ptx::fma2(make_float2(__uint_as_float(sr[2 * e2]),
                                                                    __uint_as_float(sr[2 * e2 + 1])),
                                                        make_float2(sl2, sl2), nl),
                                              e2);
                        if (decltype(masked)::value) {
                            if (r0 < lo_r || r0 >= hi_r) pv.x = 0.f;
                            if (r0 + 1 < lo_r || r0 + 1 >= hi_r) pv.y = 0.f;
                        }
                        const float2 dv = ptx::mul2(
                            pv, ptx::add2(make_float2(__uint_as_float(dr[2 * e2]), __uint_as_float(dr[2 * e2 + 1])), nd));
                        pp[e2] = ptx::pack_bf16x2(pv.x, pv.y);
                        dd[e2] = ptx::pack_bf16x2(dv.x, dv.y);
                    }
                    // chunk c's packed columns [16c, 16c+16) lie in columns
                    // this thread has already read
                    ptx::tmem_st16(tH + 16 * c, pp);
                    ptx::tmem_st16(tH + 64 + 16 * c, dd);
                }
            };
            if (all_vis) tile(std::false_type{});
            else tile(std::true_type{});
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(hs ? &bars->p_full2 : &bars->p_full);
        }
        if (ok) {
            const bool got = ptx::mbar_wait(&bars->fin, 0, p.wait_limit, abort_flag);
            if (!half_all(hs, got)) {
                flag_timeout(p.status, bars);
                ok = false;
            }
        }
        ptx::tc_fence_after();
        if (ok && depth_mode) {
            // dkd (scaled) and dvd of this chunk's depth rows, written directly
            const bool valid = j < p.T * p.Ld;
            const long long off = (((long long)b * p.T * p.Ld + (valid ? j : 0)) * p.Hkv + kvh) * kD;
            __nv_bfloat16* dvr = static_cast<__nv_bfloat16*>(p.dvd) + off;
            __nv_bfloat16* dkr = static_cast<__nv_bfloat16*>(p.dkd) + off;
#pragma unroll 1
            for (int c = 0; c < 2; ++c) {
                const int col = 64 * hs + 32 * c;  // feature columns of the chunk
                uint32_t a[32], g[32];
                ptx::tmem_ld32(tmem + lane_off + 256 + col, a);
                ptx::tmem_ld32(tmem + lane_off + 384 + col, g);
                ptx::tmem_wait_ld();
                uint32_t wa[16], wg[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    wa[e] = ptx::pack_bf16x2(__uint_as_float(a[2 * e]), __uint_as_float(a[2 * e + 1]));
                    wg[e] = ptx::pack_bf16x2(__uint_as_float(g[2 * e]) * p.scale, __uint_as_float(g[2 * e + 1]) * p.scale);
                }
                if (valid) {
                    uint4* da = reinterpret_cast<uint4*>(dvr + col);
                    uint4* dg = reinterpret_cast<uint4*>(dkr + col);
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        da[v] = make_uint4(wa[4 * v], wa[4 * v + 1], wa[4 * v + 2], wa[4 * v + 3]);
                        dg[v] = make_uint4(wg[4 * v], wg[4 * v + 1], wg[4 * v + 2], wg[4 * v + 3]);
                    }
                }
            }
        } else if (ok) {
            // This chunk's partial dK (scaled) and dV, added into the fp32
            // accumulators (other chunks of the same key tile add theirs).
            const bool valid = j < p.T;
            const long long off = (((long long)b * p.T + (valid ? j : 0)) * p.Hkv + kvh) * kD;
#pragma unroll 1
            for (int c = 0; c < 2; ++c) {
                const int col = 64 * hs + 32 * c;  // feature columns of the chunk
                uint32_t a[32], g[32];
                ptx::tmem_ld32(tmem + lane_off + 256 + col, a);
                ptx::tmem_ld32(tmem + lane_off + 384 + col, g);
                ptx::tmem_wait_ld();
                if (valid) {
#pragma unroll
                    for (int v = 0; v < 8; ++v) {
                        red_add_v4(p.dv_acc + off + col + 4 * v, __uint_as_float(a[4 * v]),
                                   __uint_as_float(a[4 * v + 1]), __uint_as_float(a[4 * v + 2]),
                                   __uint_as_float(a[4 * v + 3]));
                        red_add_v4(p.dk_acc + off + col + 4 * v, __uint_as_float(g[4 * v]) * p.scale,
                                   __uint_as_float(g[4 * v + 1]) * p.scale, __uint_as_float(g[4 * v + 2]) * p.scale,
                                   __uint_as_float(g[4 * v + 3]) * p.scale);
                    }
                }
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 512);
    }
}

// ========================================================================= dq
struct DqParams {
    CUtensorMap tm_q, tm_do, tm_k, tm_v, tm_kd, tm_vd;
    const float* lse;
    float* rowD;  // out: D = sum_j P_j dP_j per row, for the dK/dV kernels
    void* dq;     // [B,T,Hq,d] bf16
    const void* dout;  // [B,T,Hq,d] bf16 \ for D~ = <dout, out>, formed
    const void* out;   // [B,T,Hq,d] bf16 / at the start
    const unsigned long long* depth_sel;  // [B,T] slot masks or null
    int B, T, Hq, Hkv, G, n, Ld, nqt;
    float sl2, scale;
    unsigned int* status;
    unsigned int wait_limit;
};
constexpr int kDqStages = 4;  // ring of K / V tiles, one per slot
constexpr int kDqSmem = 2 * kTile + kDqStages * kTile + 256 + 2 * 128 * 4 + 1024;
static_assert(kDqSmem <= 232448, "shared memory per CTA");

// One CTA per query tile (n tokens x G heads of one kv group), latest tokens
// first. Items: the causal key tiles, then the tile's own depth chunks (rows
// t0*Ld + 128*d .. of the [B, T*Ld, Hkv, d] view, same-token mask).
//
// Row statistic D. The softmax Jacobian needs D_t = sum_j P_tj dP_tj over
// all keys of row t, which equals <dout, out> only for the exact output: the
// output the forward stored is rounded to bf16 (and was formed from bf16 P),
// and wide depth keys amplify that rounding through dq = scale sum dS k by
// |kd|. This kernel sees every key of its rows, so it computes D itself:
// with the estimate D~ = <dout, out> (formed from the stored output at the
// start) it forms dS~ = P (dP - D~) in fp32 and accumulates, per row,
//   delta = sum_j dS~_j   (= D - D~, since sum_j P_j = 1),
//   dQ~  += dS~ K          (bf16 dS~: the near-cancellation dP - D~ is fp32)
//   Bq   += P K            (the attention-weighted mean key)
// and writes dq = scale (dQ~ - delta Bq), i.e. scale sum_j P_j (dP_j - D) k_j,
// and D = D~ + delta for the dK/dV kernels, which run after this one.
//
// Depth items carry dS~ as two bf16 terms, hi = bf16(dS~) and lo =
// bf16(dS~ - hi) (16 significant bits): depth keys are where MoDA's wide
// logits live (a token's earlier layers), and there a few large dS~ times
// large |kd| would otherwise put the bf16 rounding of dS~ (2^-9 relative)
// straight into dq. It costs 8 MMAs per depth item (one or two per tile).
//
// TMEM: R0 | R1 (S and dP alternate between them) | dQ~ | Bq. S(x) sits in
// R[x % 2] and dP(x) in R[(x + 1) % 2]. The compute warps write P(x) and
// dS~(x) in bf16 over S(x) (each column half: dS~ at its columns 0-31, P at
// 32-63; for a depth item the lo term of dS~ over the half's dP columns
// 0-31, already read). Each compute warp publishes P(x) (p_ready) before it
// reads dP(x). The MMA warp issues, in this order (tcgen05.mma operations of
// one CTA execute in issue order):
//   S(x+1) = Q K(x+1)^T   into R[(x+1) % 2], as soon as the compute warps
//                         have loaded dP(x) from there (dp_read, before they
//                         form dS~(x))
//   Bq    += P(x) K(x)    A = P(x) from R[x % 2], while dS~(x) is formed
//   dQ~   += dS~(x) K(x)  A = dS~(x) from R[x % 2], once it is written (p_full)
//   dP(x+1) = dO V(x+1)^T into R[x % 2], after both have read it
// so S(x+1) and Bq run while the compute warps form dS~(x), and the compute
// warps exponentiate S(x+1) while dQ~ and dP(x+1) run. A depth item issues
// dQ~ += lo(x) K(x) (A from R[(x+1) % 2]) after dQ~, and S(x+1) only after
// that.
// Measured against two other arrangements on the wide-GQA workload (8192
// tokens, G = 32): S(x+1) only after dS~(x) (1.23 ms) and P / dS~ in shared
// memory with SS MMAs and dO in TMEM (1.42 ms) against 1.21 ms for this one.
__global__ void __launch_bounds__(kThreads, 1) moda_bwd_dq_kernel(const __grid_constant__ DqParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;
    uint8_t* sDO = smem + kTile;
    uint8_t* sRing = smem + 2 * kTile;
    Bars* bars = reinterpret_cast<Bars*>(sRing + kDqStages * kTile);
    float* sDelta = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + 256);  // [2 halves][128 rows]

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    volatile int* abort_flag = &bars->abort_flag;
    const int bh = blockIdx.x % (p.B * p.Hkv);
    const int qt = p.nqt - 1 - blockIdx.x / (p.B * p.Hkv);  // latest tokens (most keys) first
    const int b = bh / p.Hkv, kvh = bh % p.Hkv;
    const int n = p.n;
    const int t0 = qt * n;
    const int nv = min(n, p.T - t0);                   // tokens of the tile inside the sequence
    const int n_kv = (t0 + nv - 1) / kBK + 1;
    const int n_dep = (nv * p.Ld + kBK - 1) / kBK;
    const int n_items = n_kv + n_dep;

    if (threadIdx.x == 0) init_bars(bars, kDqStages, kComputeThreads / 32);
    if (warp == 0) {
        ptx::tmem_alloc(&bars->tmem_base, 512);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
        return __all_sync(0xffffffffu, ptx::mbar_wait(bar, parity, p.wait_limit, abort_flag));
    };
    auto wait_one = [&](uint64_t* bar, uint32_t parity) {
        return ptx::mbar_wait(bar, parity, p.wait_limit, abort_flag);
    };

    if (warp == kProducerWarp) {
        const uint32_t lead = lane == 0;
        if (lead) {
            ptx::prefetch_tmap(&p.tm_q);
            ptx::prefetch_tmap(&p.tm_do);
            ptx::prefetch_tmap(&p.tm_k);
            ptx::prefetch_tmap(&p.tm_v);
            if (p.Ld > 0) {
                ptx::prefetch_tmap(&p.tm_kd);
                ptx::prefetch_tmap(&p.tm_vd);
            }
        }
        ptx::mbar_arrive_expect_tx_lead(&bars->kv_full, 2 * kTile, lead);
        for (int hf = 0; hf < 2; ++hf) {
            ptx::tma_load_4d_lead(sQ + hf * kHalf, &p.tm_q, &bars->kv_full, hf * 64, kvh * p.G, t0, b, lead);
            ptx::tma_load_4d_lead(sDO + hf * kHalf, &p.tm_do, &bars->kv_full, hf * 64, kvh * p.G, t0, b, lead);
        }
        int seq = 0;
        bool ok = true;
        for (int x = 0; x < n_items && ok; ++x) {
            for (int kv = 0; kv < 2; ++kv, ++seq) {
                const int st = seq % kDqStages;
                if (!wait_all(&bars->empty[st], ((seq / kDqStages) & 1) ^ 1)) {
                    if (lead) flag_timeout(p.status, bars);
                    ok = false;
                    break;
                }
                ptx::mbar_arrive_expect_tx_lead(&bars->full[st], kTile, lead);
                uint8_t* dst = sRing + st * kTile;
                for (int hf = 0; hf < 2; ++hf) {
                    if (x < n_kv)
                        ptx::tma_load_4d_lead(dst + hf * kHalf, kv ? &p.tm_v : &p.tm_k, &bars->full[st], hf * 64,
                                              kvh, x * kBK, b, lead);
                    else
                        ptx::tma_load_4d_lead(dst + hf * kHalf, kv ? &p.tm_vd : &p.tm_kd, &bars->full[st], hf * 64,
                                              kvh, t0 * p.Ld + (x - n_kv) * kBK, b, lead);
                }
            }
        }
        ptx::mbar_wait(&bars->kv_full, 0, 0, nullptr);
        for (int s = (seq > kDqStages ? seq - kDqStages : 0); s < seq; ++s)
            ptx::mbar_wait(&bars->full[s % kDqStages], (s / kDqStages) & 1, 0, nullptr);
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // One thread runs the MMA schedule (a single-thread tcgen05.mma issue
        // costs about 60 cycles, a warp-wide one predicated on one lane 80-90,
        // against 64 cycles of tensor work for a 128x128x16 MMA; measured on
        // the B200).
        if (lane == 0) {
            constexpr uint32_t idesc_ss = ptx::idesc_bf16_f32(128, 128, 0, 0);
            constexpr uint32_t idesc_ts = ptx::idesc_bf16_f32(128, kD, 0, 1);
            const uint64_t dQk = kdesc(ptx::smem_u32(sQ)), dOk = kdesc(ptx::smem_u32(sDO));
            const uint32_t aRing = ptx::smem_u32(sRing);
            bool ok = wait_one(&bars->kv_full, 0);
            if (!ok) flag_timeout(p.status, bars);
            ptx::tc_fence_after();
            // ring slots: item x has K at 2x, V at 2x+1
            auto issue_s = [&](int x) {  // S(x) = Q K(x)^T into R[x % 2]
                const int sk = 2 * x;
                if (!wait_one(&bars->full[sk % kDqStages], (sk / kDqStages) & 1)) return false;
                ptx::tc_fence_after();
                const uint64_t kk = kdesc(aRing + (sk % kDqStages) * kTile);
#pragma unroll
                for (int k = 0; k < kD / 16; ++k)
                    ptx::mma_ss(tmem + (x & 1) * 128, dQk + koff(k), kk + koff(k), idesc_ss, k > 0);
                ptx::mma_commit(&bars->s_full);
                return true;
            };
            auto issue_dp = [&](int x) {  // dP(x) = dO V(x)^T into R[(x + 1) % 2]
                const int sv = 2 * x + 1;
                if (!wait_one(&bars->full[sv % kDqStages], (sv / kDqStages) & 1)) return false;
                ptx::tc_fence_after();
                const uint64_t vk = kdesc(aRing + (sv % kDqStages) * kTile);
#pragma unroll
                for (int k = 0; k < kD / 16; ++k)
                    ptx::mma_ss(tmem + ((x + 1) & 1) * 128, dOk + koff(k), vk + koff(k), idesc_ss, k > 0);
                ptx::mma_commit(&bars->dp_full);
                return true;
            };
            if (ok) ok = issue_s(0) && issue_dp(0);
            for (int x = 0; x < n_items && ok; ++x) {
                // the compute warps have read dP(x) from R[(x + 1) % 2], which
                // S(x + 1) may now overwrite (depth items: after the lo MMA);
                // each warp published P(x) before it read dP(x), so p_ready
                // has completed too (and cannot run a phase ahead: P(x+1)
                // needs S(x+1), issued below)
                if (!wait_one(&bars->dp_read, x & 1) || !wait_one(&bars->p_ready, x & 1)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const bool depth_item = x >= n_kv;
                if (!depth_item && x + 1 < n_items && !issue_s(x + 1)) {
                    ok = false;
                    break;
                }
                const int sk = 2 * x;
                const uint64_t km = mndesc(aRing + (sk % kDqStages) * kTile);
                // Bq += P(x) K(x) while the compute warps form dS~(x)
#pragma unroll
                for (int k = 0; k < kBK / 16; ++k)
                    ptx::mma_ts(tmem + 384, tmem + (x & 1) * 128 + 32 + acol(k), km + mnoff(k), idesc_ts,
                                     (x > 0 || k > 0) ? 1u : 0u);
                if (!wait_one(&bars->p_full, x & 1)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
#pragma unroll
                for (int k = 0; k < kBK / 16; ++k)
                    ptx::mma_ts(tmem + 256, tmem + (x & 1) * 128 + acol(k), km + mnoff(k), idesc_ts,
                                     (x > 0 || k > 0) ? 1u : 0u);
                if (depth_item) {
                    // the lo term of dS~(x), then S(x + 1) over it
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k)
                        ptx::mma_ts(tmem + 256, tmem + ((x + 1) & 1) * 128 + acol(k), km + mnoff(k), idesc_ts, 1u);
                    if (x + 1 < n_items && !issue_s(x + 1)) {
                        ok = false;
                        break;
                    }
                }
                // K(x), V(x) are no longer needed
                ptx::mma_commit(&bars->empty[sk % kDqStages]);
                ptx::mma_commit(&bars->empty[(sk + 1) % kDqStages]);
                // dP(x + 1) into R[x % 2], after dQ~ and Bq have read it
                if (x + 1 < n_items && !issue_dp(x + 1)) {
                    ok = false;
                    break;
                }
            }
            if (!ok) flag_timeout(p.status, bars);
            if (ok) ptx::mma_commit(&bars->fin);
            ptx::mma_commit(&bars->drain);
            ptx::mbar_wait(&bars->drain, 0, 0, nullptr);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ compute warps
        // Column half hs: key columns 64hs .. 64hs+63 of S / dP, and feature
        // columns 64hs .. of dQ in the epilogue.
        const int hs = warp / 4;
        const int r = (warp % 4) * 32 + lane;  // TMEM lane = query row (token-major)
        const uint32_t lane_off = (uint32_t)((warp % 4) * 32) << 16;
        const int tt = r / p.G;          // token within the tile
        const int t = t0 + tt, h = kvh * p.G + r % p.G;
        const bool row_ok = t < p.T;
        float lse2 = INFINITY;
        if (row_ok) lse2 = p.lse[((long long)b * p.Hq + h) * p.T + t] * kLog2e;
        // D~ = <dout, out> of the row from the stored output: each column half
        // sums its 64 features, and the halves add through shared memory
        // (sDelta is written again only after the item loop, which no thread
        // finishes before every thread has passed this point: each item
        // needs the arrivals of all 256 compute threads)
        float Drow;
        {
            const long long roff = (((long long)b * p.T + (row_ok ? t : 0)) * p.Hq + h) * kD + 64 * hs;
            const uint4* du = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.dout) + roff);
            const uint4* ou = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.out) + roff);
            float part = 0.f;
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                const uint4 u = row_ok ? du[v] : make_uint4(0u, 0u, 0u, 0u);
                const uint4 o = row_ok ? ou[v] : make_uint4(0u, 0u, 0u, 0u);
                const uint32_t uw[4] = {u.x, u.y, u.z, u.w}, ow[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    part = fmaf(__uint_as_float(uw[q] << 16), __uint_as_float(ow[q] << 16), part);
                    part = fmaf(__uint_as_float(uw[q] & 0xffff0000u), __uint_as_float(ow[q] & 0xffff0000u), part);
                }
            }
            sDelta[hs * 128 + r] = part;
            asm volatile("bar.sync 1, %0;" ::"n"(kComputeThreads) : "memory");
            Drow = sDelta[r] + sDelta[128 + r];
        }
        const float sl2 = p.sl2;
        const bool has_sel = p.depth_sel != nullptr;
        const unsigned long long sel =
            has_sel && row_ok ? p.depth_sel[(long long)b * p.T + t] & depth_slot_bits(p.Ld) : 0ull;
        float delta = 0.f;  // sum of this half's dS~ over every item (fp32)
        bool ok = true;
        for (int x = 0; x < n_items; ++x) {
            const uint32_t rS = tmem + lane_off + (x & 1) * 128;        // S(x), then dS(x)
            const uint32_t rP = tmem + lane_off + ((x + 1) & 1) * 128;  // dP(x)
            if (!__all_sync(0xffffffffu, ptx::mbar_wait(&bars->s_full, x & 1, p.wait_limit, abort_flag))) {
                flag_timeout(p.status, bars);
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            float pr[64];  // P of this half's 64 key columns
            {
                uint32_t su[64];
#pragma unroll
                for (int c = 0; c < 2; ++c)
                    ptx::tmem_ld32(rS + 64 * hs + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&su[c * 32]));
                ptx::tmem_wait_ld();
                // a key tile wholly at or before every row of the warp needs no
                // mask (warp-uniform test; x < n_kv is the same for the warp)
                const bool all_vis = x < n_kv && __all_sync(0xffffffffu, x * kBK + 64 * hs + 63 <= t);
                if (all_vis) {
                    const float2 sl2x2 = make_float2(sl2, sl2), nl2x2 = make_float2(-lse2, -lse2);
#pragma unroll
                    for (int c = 0; c < 64; c += 2) {
                        const float2 e = exp2_pair(
                            ptx::fma2(make_float2(__uint_as_float(su[c]), __uint_as_float(su[c + 1])), sl2x2, nl2x2),
                            c / 2);
                        pr[c] = e.x;
                        pr[c + 1] = e.y;
                    }
                } else {
                    uint32_t vis[4];  // visible columns of this row
                    if (x < n_kv)
                        depth_col_mask(0, t - x * kBK + 1, false, 0ull, vis);  // keys <= t
                    else  // the row's own depth rows (selected slots)
                        depth_col_mask(tt * p.Ld - (x - n_kv) * kBK, p.Ld, has_sel, sel, vis);
                    const uint32_t vw[2] = {hs ? vis[2] : vis[0], hs ? vis[3] : vis[1]};
#pragma unroll
                    for (int c = 0; c < 64; c += 2) {
                        const float2 e = exp2_pair(make_float2(fmaf(__uint_as_float(su[c]), sl2, -lse2),
                                                               fmaf(__uint_as_float(su[c + 1]), sl2, -lse2)),
                                                   c / 2);
                        pr[c] = ((vw[c >> 5] >> (c & 31)) & 1u) ? e.x : 0.f;
                        pr[c + 1] = ((vw[c >> 5] >> ((c + 1) & 31)) & 1u) ? e.y : 0.f;
                    }
                }
                // P in bf16 over this half's S columns 32-63 (already read)
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t pp[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) pp[e] = ptx::pack_bf16x2(pr[32 * c + 2 * e], pr[32 * c + 2 * e + 1]);
                    ptx::tmem_st16(rS + 64 * hs + 32 + 16 * c, pp);
                }
                // P is in TMEM: Bq += P K may go out before dS~ is formed
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&bars->p_ready);
            }
            if (!__all_sync(0xffffffffu, ptx::mbar_wait(&bars->dp_full, x & 1, p.wait_limit, abort_flag))) {
                flag_timeout(p.status, bars);
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            const bool depth_item = x >= n_kv;
            uint32_t drr[64];
#pragma unroll
            for (int c = 0; c < 2; ++c)
                ptx::tmem_ld32(rP + 64 * hs + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&drr[32 * c]));
            ptx::tmem_wait_ld();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&bars->dp_read);
            // dS~ in bf16 (hi), and for a depth item also the lo term (two loop
            // versions: the lo arithmetic only where it is stored); packed fp32
            // pairs, the row sum of dS~ in two lanes
            const float2 nDrow = make_float2(-Drow, -Drow);
            float2 dsum = make_float2(0.f, 0.f);
            auto ds_pass = [&](auto with_lo) {
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const uint32_t* dr = drr + 32 * c;
                    uint32_t dd[16], dl[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float2 d = ptx::mul2(
                            make_float2(pr[32 * c + 2 * e], pr[32 * c + 2 * e + 1]),
                            ptx::add2(make_float2(__uint_as_float(dr[2 * e]), __uint_as_float(dr[2 * e + 1])), nDrow));
                        dsum = ptx::add2(dsum, d);
                        const float d0 = d.x, d1 = d.y;
                        dd[e] = ptx::pack_bf16x2(d0, d1);
                        // lo term: the part of dS~ the bf16 hi term drops
                        if (decltype(with_lo)::value)
                            dl[e] = ptx::pack_bf16x2(d0 - __uint_as_float(dd[e] << 16),
                                                     d1 - __uint_as_float(dd[e] & 0xffff0000u));
                    }
                    ptx::tmem_st16(rS + 64 * hs + 16 * c, dd);  // over this half's S(x), already read
                    // over this half's dP(x) columns 16c.., read in chunk 0
                    if (decltype(with_lo)::value) ptx::tmem_st16(rP + 64 * hs + 16 * c, dl);
                }
            };
            if (depth_item) ds_pass(std::true_type{});
            else ds_pass(std::false_type{});
            delta += dsum.x + dsum.y;
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&bars->p_full);
        }
        if (ok && !__all_sync(0xffffffffu, ptx::mbar_wait(&bars->fin, 0, p.wait_limit, abort_flag))) {
            flag_timeout(p.status, bars);
            ok = false;
        }
        ptx::tc_fence_after();
        // delta of the whole row = the two column halves' sums (every
        // compute thread reaches this barrier, whether or not ok)
        sDelta[hs * 128 + r] = delta;
        asm volatile("bar.sync 1, %0;" ::"n"(kComputeThreads) : "memory");
        delta = sDelta[r] + sDelta[128 + r];
        if (ok) {
            if (row_ok && hs == 0) p.rowD[((long long)b * p.Hq + h) * p.T + t] = Drow + delta;
            __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.dq) + (((long long)b * p.T + (row_ok ? t : 0)) * p.Hq + h) * kD;
            const float nds = -delta;
#pragma unroll 1
            for (int c = 0; c < 2; ++c) {
                const int col = 64 * hs + 32 * c;  // feature columns of the chunk
                uint32_t o[32], bq[32];
                ptx::tmem_ld32(tmem + lane_off + 256 + col, o);
                ptx::tmem_ld32(tmem + lane_off + 384 + col, bq);
                ptx::tmem_wait_ld();
                uint32_t w[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float g0 = fmaf(nds, __uint_as_float(bq[2 * e]), __uint_as_float(o[2 * e]));
                    const float g1 = fmaf(nds, __uint_as_float(bq[2 * e + 1]), __uint_as_float(o[2 * e + 1]));
                    w[e] = ptx::pack_bf16x2(g0 * p.scale, g1 * p.scale);
                }
                if (row_ok) {
                    uint4* d4 = reinterpret_cast<uint4*>(dst + col);
#pragma unroll
                    for (int v = 0; v < 4; ++v) d4[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
                }
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 512);
    }
}

// fp32 accumulator -> bf16 (dk, dv).
__global__ void acc_to_bf16_kernel(const float4* acc, uint2* out, long long n4) {
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
         i += (long long)gridDim.x * blockDim.x) {
        const float4 v = acc[i];
        out[i] = make_uint2(ptx::pack_bf16x2(v.x, v.y), ptx::pack_bf16x2(v.z, v.w));
    }
}

int sm_count() {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

}  // namespace

bool bwd_tc_supported(const BwdArgs& a) {
    const FwdArgs& f = a.f;
    if (f.dtype != MODA_BF16 || f.d != kD) return false;
    if (f.G < 1 || f.G > 128 || 128 % f.G) return false;
    if (!a.dk_acc || !a.dv_acc) return false;
    if ((long long)f.T * f.Ld >= (1LL << 31)) return false;
    const Strides4 sq = strides_q(f.T, f.Hq, f.d), skv = strides_q(f.T, f.Hkv, f.d);
    const Strides5 sdep = strides_depth_native(f.T, f.Ld, f.Hkv, f.d);
    if (f.sq.sb != sq.sb || f.sq.st != sq.st || f.sq.sh != sq.sh) return false;
    if (f.skv.sb != skv.sb || f.skv.st != skv.st || f.skv.sh != skv.sh) return false;
    if (f.Ld > 0 && (f.sdep.sb != sdep.sb || f.sdep.st != sdep.st || f.sdep.si != sdep.si ||
                     f.sdep.sh != sdep.sh))
        return false;
    return true;
}

cudaError_t launch_bwd_tc(const BwdArgs& a, cudaStream_t s) {
    const FwdArgs& f = a.f;
    cudaError_t e;
    const int G = f.G, n = 128 / G;
    int gshift = 0;
    while ((1 << gshift) < G) ++gshift;
    const cuuint64_t es = 2;
    CUtensorMap tm_q, tm_do, tm_k, tm_v, tm_kd, tm_vd;
    {
        const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)f.Hq, (cuuint64_t)f.T, (cuuint64_t)f.B};
        const cuuint64_t st[3] = {kD * es, (cuuint64_t)f.Hq * kD * es, (cuuint64_t)f.T * f.Hq * kD * es};
        const cuuint32_t box[4] = {64, (cuuint32_t)G, (cuuint32_t)n, 1};
        if (!make_tmap_bf16_4d(&tm_q, f.q, dims, st, box)) return cudaErrorInvalidValue;
        if (!make_tmap_bf16_4d(&tm_do, a.dout, dims, st, box)) return cudaErrorInvalidValue;
    }
    {
        const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)f.Hkv, (cuuint64_t)f.T, (cuuint64_t)f.B};
        const cuuint64_t st[3] = {kD * es, (cuuint64_t)f.Hkv * kD * es, (cuuint64_t)f.T * f.Hkv * kD * es};
        const cuuint32_t box[4] = {64, 1, (cuuint32_t)kBK, 1};
        if (!make_tmap_bf16_4d(&tm_k, f.k, dims, st, box)) return cudaErrorInvalidValue;
        if (!make_tmap_bf16_4d(&tm_v, f.v, dims, st, box)) return cudaErrorInvalidValue;
    }
    if (f.Ld > 0) {
        const cuuint64_t rows = (cuuint64_t)f.T * f.Ld;
        const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)f.Hkv, rows, (cuuint64_t)f.B};
        const cuuint64_t st[3] = {kD * es, (cuuint64_t)f.Hkv * kD * es, rows * f.Hkv * kD * es};
        const cuuint32_t box[4] = {64, 1, (cuuint32_t)kBK, 1};
        if (!make_tmap_bf16_4d(&tm_kd, f.kd, dims, st, box)) return cudaErrorInvalidValue;
        if (!make_tmap_bf16_4d(&tm_vd, f.vd, dims, st, box)) return cudaErrorInvalidValue;
    } else {
        tm_kd = tm_k;
        tm_vd = tm_v;
    }
    const int sms = sm_count();

    // ---- dq (first: it turns rowD into the exact D the dK/dV kernels read)
    DqParams pq;
    memset(&pq, 0, sizeof(pq));
    pq.tm_q = tm_q; pq.tm_do = tm_do; pq.tm_k = tm_k; pq.tm_v = tm_v; pq.tm_kd = tm_kd; pq.tm_vd = tm_vd;
    pq.lse = f.lse; pq.rowD = a.rowD; pq.dq = a.dq; pq.dout = a.dout; pq.out = f.out;
    pq.B = f.B; pq.T = f.T; pq.Hq = f.Hq; pq.Hkv = f.Hkv; pq.G = G; pq.n = n; pq.Ld = f.Ld;
    pq.nqt = (f.T + n - 1) / n;
    pq.depth_sel = f.depth_sel;
    pq.sl2 = f.scale * kLog2e; pq.scale = f.scale;
    pq.status = f.status; pq.wait_limit = f.wait_limit;
    if ((e = cudaFuncSetAttribute(moda_bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDqSmem)) !=
        cudaSuccess)
        return e;
    const long long grid_q = (long long)pq.nqt * f.B * f.Hkv;
    if (grid_q > 0x7fffffffLL) return cudaErrorInvalidValue;
    moda_bwd_dq_kernel<<<(unsigned)grid_q, kThreads, kDqSmem, s>>>(pq);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    // ---- dk, dv
    DkvParams pk;
    memset(&pk, 0, sizeof(pk));
    pk.tm_q = tm_q; pk.tm_do = tm_do; pk.tm_k = tm_k; pk.tm_v = tm_v; pk.tm_kd = tm_kd; pk.tm_vd = tm_vd;
    pk.lse = f.lse; pk.rowD = a.rowD; pk.dk_acc = a.dk_acc; pk.dv_acc = a.dv_acc;
    pk.B = f.B; pk.T = f.T; pk.Hq = f.Hq; pk.Hkv = f.Hkv; pk.G = G; pk.n = n; pk.gshift = gshift;
    pk.sl2 = f.scale * kLog2e; pk.scale = f.scale;
    pk.status = f.status; pk.wait_limit = f.wait_limit;
    const int nkt = (f.T + kBK - 1) / kBK;
    {
        // query tiles per CTA: ~4 waves over the SMs, at least 16 tiles each
        long long steps = 0;
        for (int kt = 0; kt < nkt; ++kt) steps += (f.T - kt * kBK + n - 1) / n;
        steps *= (long long)f.B * f.Hkv;
        long long qc = (steps + 4LL * sms - 1) / (4LL * sms);
        pk.qchunk = (int)(qc < 16 ? 16 : qc);
    }
    const size_t kv_bytes = (size_t)f.B * f.T * f.Hkv * kD * sizeof(float);
    if ((e = cudaMemsetAsync(a.dk_acc, 0, kv_bytes, s)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(a.dv_acc, 0, kv_bytes, s)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(moda_bwd_dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDkvSmem)) !=
        cudaSuccess)
        return e;
    // sequence-mode CTAs (key tile, chunk of query tokens, (b, kv-head)), then
    // with depth keys the depth-mode CTAs (128-row depth chunk, (b, kv-head))
    pk.nkt = nkt;
    pk.n_chunks = ((f.T + n - 1) / n + pk.qchunk - 1) / pk.qchunk;
    pk.n_seq_ctas = (long long)nkt * pk.n_chunks * f.B * f.Hkv;
    long long grid_kv = pk.n_seq_ctas;
    if (f.Ld > 0) {
        const long long chunks = ((long long)f.T * f.Ld + kBK - 1) / kBK;
        if (chunks > 0x7fffffffLL) return cudaErrorInvalidValue;
        pk.n_dep_chunks = (int)chunks;
        pk.Ld = f.Ld;
        pk.depth_sel = f.depth_sel;
        pk.dkd = a.dkd;
        pk.dvd = a.dvd;
        grid_kv += chunks * f.B * f.Hkv;
    }
    if (grid_kv > 0x7fffffffLL) return cudaErrorInvalidValue;
    moda_bwd_dkdv_kernel<<<(unsigned)grid_kv, kThreads, kDkvSmem, s>>>(pk);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    // ---- dk, dv to bf16
    const long long n4 = (long long)f.B * f.T * f.Hkv * kD / 4;
    long long blocks = (n4 + 255) / 256;
    if (blocks > (long long)sms * 8) blocks = (long long)sms * 8;
    acc_to_bf16_kernel<<<(unsigned)blocks, 256, 0, s>>>(reinterpret_cast<const float4*>(a.dk_acc),
                                                        static_cast<uint2*>(a.dk), n4);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    acc_to_bf16_kernel<<<(unsigned)blocks, 256, 0, s>>>(reinterpret_cast<const float4*>(a.dv_acc),
                                                        static_cast<uint2*>(a.dv), n4);
    return cudaGetLastError();
}

}  // namespace moda
