// Tensor-core MoDA backward for sm_100a (bf16, d = 128, 128 % G == 0).
//
// The pages give no backward pass; this computes the derivative of the MoDA
// forward ("动态混合深度注意力机制MoDA技术解析" (mhpn.cn) §1.2 formula, §2.2 dual
// mask) with the usual softmax-Jacobian identities:
//   P = exp(s - lse),  D = <dout, out>,  dS = P * (dP - D),  dP = dout . v
//   dq = scale (sum_j dS_j k_j + sum_i dS'_i kd_i)
//   dk_j = scale sum dS_j q,  dv_j = sum P_j dout   (rows t >= j, G heads)
//   dkd_i = scale sum_h dS'_i q,  dvd_i = sum_h P'_i dout   (same token)
//
// Launch sequence (one stream):
//   1. D = rowsum(dout * out)                      (SIMT, shared with the SIMT path)
//   2. dq_acc = scale * sum_i dS'_i kd_i            (SIMT; plain store, 0 when Ld = 0)
//   3. dkd, dvd                                     (SIMT, shared with the SIMT path)
//   4. sequence part, KV-major, tensor cores        (this file): dq, dk and dv
//      partials added into fp32 accumulators with vector fp32 reductions
//   5. dq, dk, dv = bf16(accumulators)
//
// Kernel 4: one CTA per (b, kv-head, 128-key tile, chunk of query tiles); it
// walks its share of the query tiles of the rows that can see its keys
// (tokens t >= j0), 128 rows each in the
// forward's token-major GQA order (n = 128 / G tokens x G heads), so the
// G heads' contributions to dk / dv sum inside the TMEM accumulators.
// Per query tile:
//   S^T  = K Q^T   and   dP^T = V dO^T          (SS MMAs -> TMEM)
//   CUDA cores (one thread per key): P^T, dS^T -> bf16 -> TMEM (over S^T and
//   dP^T) for the next two MMAs, and dS -> shared memory for the third
//   dV += P^T dO,  dK += dS^T Q                  (A operand from TMEM)
//   dQ_tile = dS K                               (A from shared memory) -> TMEM
//   CUDA cores (one thread per query row): red.global.add.v4.f32 into dq_acc.
// TMEM: S^T | dP^T | dV | dK (128 fp32 columns each); dQ_tile reuses S^T's
// columns once dV has read P^T (tcgen05.mma of one thread run in order).
#include <cuda_bf16.h>

#include <cmath>
#include <cstring>

#include "moda_internal.h"
#include "sm100_ptx.cuh"
#include "tmap_host.h"

namespace moda {
namespace {

constexpr int kD = 128;
constexpr int kBK = 128;          // keys per CTA
constexpr int kStages = 2;        // query-tile ring (Q and dO per stage)
constexpr int kTile = 128 * kD * 2;
constexpr int kHalf = kTile / 2;
constexpr int kThreads = 192;     // warps 0-3 compute, 4 TMA producer, 5 MMA
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr float kLog2e = 1.4426950408889634f;

struct TcBwdParams {
    CUtensorMap tm_q, tm_do, tm_k, tm_v;
    const float* lse;
    const float* rowD;
    float* dq_acc;
    float* dk_acc;  // [B,T,Hkv,d] fp32, zeroed before the launch
    float* dv_acc;
    int B, T, Hq, Hkv, G, n, nkt, qchunk;
    float sl2, scale;
    unsigned int* status;
    unsigned int wait_limit;
};

struct __align__(8) Bars {
    uint64_t kv_full;
    uint64_t qd_full[kStages];
    uint64_t qd_empty[kStages];
    uint64_t s_full, p_full, dq_full, tmem_free, fin, drain;
    uint32_t tmem_base;
    int abort_flag;
};

// K, V, ring of (Q, dO), dS, then the tile's lse / D and the barriers.
constexpr int kSmemBytes = 2 * kTile + kStages * 2 * kTile + kTile + 2 * 128 * 4 + 128 + 1024;
static_assert(sizeof(Bars) <= 128, "barrier block");
static_assert(kSmemBytes <= 232448, "shared memory per CTA");

__device__ __forceinline__ uint64_t desc_k(uint32_t tile, int k16) {
    return ptx::umma_desc_sw128(tile + (k16 >> 2) * kHalf + (k16 & 3) * 32, 16, 1024);
}
__device__ __forceinline__ uint64_t desc_mn(uint32_t tile, int k16) {
    return ptx::umma_desc_sw128(tile + k16 * 16 * 128, kHalf, 1024);
}

__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}
// Barrier 1 spans the 128 compute threads only.
__device__ __forceinline__ void named_sync_compute() {
    asm volatile("bar.sync 1, 128;" ::: "memory");
}
// AND of `v` over the 128 compute threads (a barrier too): every compute
// warp takes the same branch after a bounded wait, so none is left waiting at
// a later named barrier.
__device__ __forceinline__ bool all_compute(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.and.pred po, 1, 128, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void flag_timeout(TcBwdParams const& p, Bars* bars) {
    *reinterpret_cast<volatile int*>(&bars->abort_flag) = 1;
    atomicOr(p.status, 1u);
}

__global__ void __launch_bounds__(kThreads, 1) moda_bwd_seq_tc_kernel(const __grid_constant__ TcBwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sK = smem;
    uint8_t* sV = smem + kTile;
    uint8_t* sRing = smem + 2 * kTile;                  // stage s: Q at +2s*kTile, dO at +(2s+1)*kTile
    uint8_t* sDS = sRing + kStages * 2 * kTile;
    float* sStat = reinterpret_cast<float*>(sDS + kTile);  // [lse2 128 | D 128] of the query tile
    Bars* bars = reinterpret_cast<Bars*>(sStat + 256);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const uint32_t wait_limit = p.wait_limit;
    volatile int* abort_flag = &bars->abort_flag;

    // Work item: key tile = blockIdx.x (fastest), chunk of query tokens =
    // blockIdx.y, (b, kv-head) = blockIdx.z. A chunk is qchunk query tiles of
    // absolute token range [c*qchunk*n, (c+1)*qchunk*n); the CTAs in flight
    // at one time are the key tiles of one or two chunks, so their fp32 dq
    // reductions land on the same few MB of dq rows (L2-resident). Key tiles
    // that no row of the chunk can see exit at once.
    const int b = blockIdx.z / p.Hkv, kvh = blockIdx.z % p.Hkv;
    const int kt = blockIdx.x;
    const int j0 = kt * kBK;
    const int n = p.n;
    const int c_lo = blockIdx.y * p.qchunk * n;                      // first token of the chunk
    const int c_hi = min(p.T, (blockIdx.y + 1) * p.qchunk * n);      // one past its last token
    const int t_first = max(j0, c_lo);                               // multiple of n
    if (t_first >= c_hi) return;
    const int nq = (c_hi - t_first + n - 1) / n;
    const int q_first = (t_first - j0) / n;                          // query tiles counted from j0

    if (threadIdx.x == 0) {
        ptx::mbar_init(&bars->kv_full, 1);
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(&bars->qd_full[s], 1);
            ptx::mbar_init(&bars->qd_empty[s], 1);
        }
        ptx::mbar_init(&bars->s_full, 1);
        ptx::mbar_init(&bars->p_full, 128);
        ptx::mbar_init(&bars->dq_full, 1);
        ptx::mbar_init(&bars->tmem_free, 128);
        ptx::mbar_init(&bars->fin, 1);
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

    if (warp == kProducerWarp) {
        if (lane == 0) {
            ptx::prefetch_tmap(&p.tm_q);
            ptx::prefetch_tmap(&p.tm_do);
            ptx::prefetch_tmap(&p.tm_k);
            ptx::prefetch_tmap(&p.tm_v);
            ptx::mbar_arrive_expect_tx(&bars->kv_full, 2 * kTile);
            for (int hf = 0; hf < 2; ++hf) {
                ptx::tma_load_4d(sK + hf * kHalf, &p.tm_k, &bars->kv_full, hf * 64, kvh, j0, b);
                ptx::tma_load_4d(sV + hf * kHalf, &p.tm_v, &bars->kv_full, hf * 64, kvh, j0, b);
            }
            int issued = 0;
            for (int i = 0; i < nq; ++i) {
                const int st = i % kStages;
                const uint32_t ph = (i / kStages) & 1;
                if (!ptx::mbar_wait(&bars->qd_empty[st], ph ^ 1, wait_limit, abort_flag)) {
                    flag_timeout(p, bars);
                    break;
                }
                ptx::mbar_arrive_expect_tx(&bars->qd_full[st], 2 * kTile);
                uint8_t* q_dst = sRing + (2 * st) * kTile;
                uint8_t* do_dst = sRing + (2 * st + 1) * kTile;
                const int tq0 = j0 + (q_first + i) * n;
                for (int hf = 0; hf < 2; ++hf) {
                    ptx::tma_load_4d(q_dst + hf * kHalf, &p.tm_q, &bars->qd_full[st], hf * 64, kvh * p.G, tq0, b);
                    ptx::tma_load_4d(do_dst + hf * kHalf, &p.tm_do, &bars->qd_full[st], hf * 64, kvh * p.G, tq0, b);
                }
                issued = i + 1;
            }
            // Drain: every load issued lands before the CTA exits.
            ptx::mbar_wait(&bars->kv_full, 0, 0, nullptr);
            for (int i = (issued > kStages ? issued - kStages : 0); i < issued; ++i)
                ptx::mbar_wait(&bars->qd_full[i % kStages], (i / kStages) & 1, 0, nullptr);
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            constexpr uint32_t idesc_ss = ptx::idesc_bf16_f32(128, 128, 0, 0);
            constexpr uint32_t idesc_ts = ptx::idesc_bf16_f32(128, kD, 0, 1);
            constexpr uint32_t idesc_dq = ptx::idesc_bf16_f32(128, kD, 1, 1);
            const uint32_t aK = ptx::smem_u32(sK), aV = ptx::smem_u32(sV), aDS = ptx::smem_u32(sDS);
            const uint32_t aRing = ptx::smem_u32(sRing);
            bool ok = ptx::mbar_wait(&bars->kv_full, 0, wait_limit, abort_flag);
            if (!ok) flag_timeout(p, bars);
            ptx::tc_fence_after();
            for (int i = 0; i < nq && ok; ++i) {
                const int st = i % kStages;
                const uint32_t aQ = aRing + (2 * st) * kTile, aDO = aRing + (2 * st + 1) * kTile;
                ok = ptx::mbar_wait(&bars->qd_full[st], (i / kStages) & 1, wait_limit, abort_flag);
                if (ok && i > 0) ok = ptx::mbar_wait(&bars->tmem_free, (i - 1) & 1, wait_limit, abort_flag);
                if (!ok) {
                    flag_timeout(p, bars);
                    break;
                }
                ptx::tc_fence_after();
#pragma unroll
                for (int k = 0; k < kD / 16; ++k)
                    ptx::mma_ss(tmem + 0, desc_k(aK, k), desc_k(aQ, k), idesc_ss, k > 0);
#pragma unroll
                for (int k = 0; k < kD / 16; ++k)
                    ptx::mma_ss(tmem + 128, desc_k(aV, k), desc_k(aDO, k), idesc_ss, k > 0);
                ptx::mma_commit(&bars->s_full);
                if (!ptx::mbar_wait(&bars->p_full, i & 1, wait_limit, abort_flag)) {
                    flag_timeout(p, bars);
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
#pragma unroll
                for (int k = 0; k < 128 / 16; ++k)
                    ptx::mma_ts(tmem + 256, tmem + 0 + k * 8, desc_mn(aDO, k), idesc_ts, (i > 0 || k > 0) ? 1u : 0u);
#pragma unroll
                for (int k = 0; k < 128 / 16; ++k)
                    ptx::mma_ts(tmem + 384, tmem + 128 + k * 8, desc_mn(aQ, k), idesc_ts, (i > 0 || k > 0) ? 1u : 0u);
#pragma unroll
                for (int k = 0; k < kBK / 16; ++k)
                    ptx::mma_ss(tmem + 0, desc_mn(aDS, k), desc_mn(aK, k), idesc_dq, k > 0);
                ptx::mma_commit(&bars->dq_full);
                ptx::mma_commit(&bars->qd_empty[st]);
            }
            if (ok) ptx::mma_commit(&bars->fin);
            ptx::mma_commit(&bars->drain);
            ptx::mbar_wait(&bars->drain, 0, 0, nullptr);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ compute warps
        const int r = warp * 32 + lane;                 // TMEM lane
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const int j = j0 + r;                           // this thread's key
        const float sl2 = p.sl2;
        bool ok = true;
        int gshift = 0;
        while ((1 << gshift) < p.G) ++gshift;
        // lse (log2 units) and D of row r of query tile i; loaded one tile
        // ahead so the global-memory latency stays off the critical path.
        auto load_stat = [&](int i, float& l2, float& dd) {
            const int t = j0 + (q_first + i) * n + (r >> gshift), h = kvh * p.G + (r & (p.G - 1));
            if (t < p.T) {
                const long long ix = ((long long)b * p.Hq + h) * p.T + t;
                l2 = p.lse[ix] * kLog2e;
                dd = p.rowD[ix];
            } else {
                l2 = INFINITY;  // rows past T: P = 0
                dd = 0.f;
            }
        };
        float nl2, nD;
        load_stat(0, nl2, nD);
        for (int i = 0; i < nq; ++i) {
            const int tq0 = j0 + (q_first + i) * n;
            float* st_lse = sStat;
            float* st_D = sStat + 128;
            named_sync_compute();  // the previous tile's readers are done
            st_lse[r] = nl2;
            st_D[r] = nD;
            if (i + 1 < nq) load_stat(i + 1, nl2, nD);
            const bool got = ptx::mbar_wait(&bars->s_full, i & 1, wait_limit, abort_flag);
            if (!all_compute(got)) {  // also publishes st_lse / st_D
                flag_timeout(p, bars);
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            // key j is visible to row rr iff j <= t(rr) = tq0 + (rr >> gshift),
            // i.e. rows rr < (j - tq0) << gshift are masked.
            const int mask_below = j > tq0 ? (j - tq0) << gshift : 0;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t sr[32], dr[32];
                ptx::tmem_ld32(tmem + lane_off + 0 + 32 * c, sr);
                ptx::tmem_ld32(tmem + lane_off + 128 + 32 * c, dr);
                ptx::tmem_wait_ld();
                uint32_t pp[16], dd[16];
#pragma unroll
                for (int e2 = 0; e2 < 16; ++e2) {
                    float pv[2], dv[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int rr = 32 * c + 2 * e2 + u;
                        float pr = ptx::ex2(fmaf(__uint_as_float(sr[2 * e2 + u]), sl2, -st_lse[rr]));
                        if (rr < mask_below) pr = 0.f;
                        pv[u] = pr;
                        dv[u] = pr * (__uint_as_float(dr[2 * e2 + u]) - st_D[rr]);
                    }
                    pp[e2] = ptx::pack_bf16x2(pv[0], pv[1]);
                    dd[e2] = ptx::pack_bf16x2(dv[0], dv[1]);
                }
                ptx::tmem_st16(tmem + lane_off + 0 + 16 * c, pp);
                ptx::tmem_st16(tmem + lane_off + 128 + 16 * c, dd);
                // dS into shared memory, [key][row] with rows contiguous (the
                // MN-major A operand of dQ = dS K), 128-byte swizzle.
                uint8_t* half = sDS + (c >> 1) * kHalf + r * 128;
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const int chunk = ((c & 1) * 4 + v) ^ (r & 7);
                    *reinterpret_cast<uint4*>(half + chunk * 16) =
                        make_uint4(dd[4 * v], dd[4 * v + 1], dd[4 * v + 2], dd[4 * v + 3]);
                }
            }
            ptx::tmem_wait_st();
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            ptx::mbar_arrive(&bars->p_full);

            // dQ tile (lane = query row) -> fp32 reductions into dq_acc.
            const bool got2 = ptx::mbar_wait(&bars->dq_full, i & 1, wait_limit, abort_flag);
            if (!all_compute(got2)) {
                flag_timeout(p, bars);
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            {
                const int t = tq0 + (r >> gshift), h = kvh * p.G + (r & (p.G - 1));
                float* dst = p.dq_acc + (((long long)b * p.T + (t < p.T ? t : 0)) * p.Hq + h) * kD;
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t o[32];
                    ptx::tmem_ld32(tmem + lane_off + 32 * c, o);
                    ptx::tmem_wait_ld();
                    if (t < p.T) {
#pragma unroll
                        for (int v = 0; v < 8; ++v)
                            red_add_v4(dst + 32 * c + 4 * v, __uint_as_float(o[4 * v]) * p.scale,
                                       __uint_as_float(o[4 * v + 1]) * p.scale, __uint_as_float(o[4 * v + 2]) * p.scale,
                                       __uint_as_float(o[4 * v + 3]) * p.scale);
                    }
                }
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(&bars->tmem_free);
        }
        if (ok) {
            const bool got = ptx::mbar_wait(&bars->fin, 0, wait_limit, abort_flag);
            if (!all_compute(got)) {
                flag_timeout(p, bars);
                ok = false;
            }
        }
        ptx::tc_fence_after();
        if (ok) {
            // This chunk's partial dK (scaled) and dV, added into the fp32
            // accumulators (other chunks of the same key tile add theirs).
            const bool valid = j < p.T;
            const long long off = (((long long)b * p.T + (valid ? j : 0)) * p.Hkv + kvh) * kD;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t a[32], g[32];
                ptx::tmem_ld32(tmem + lane_off + 256 + 32 * c, a);
                ptx::tmem_ld32(tmem + lane_off + 384 + 32 * c, g);
                ptx::tmem_wait_ld();
                if (valid) {
#pragma unroll
                    for (int v = 0; v < 8; ++v) {
                        red_add_v4(p.dv_acc + off + 32 * c + 4 * v, __uint_as_float(a[4 * v]),
                                   __uint_as_float(a[4 * v + 1]), __uint_as_float(a[4 * v + 2]),
                                   __uint_as_float(a[4 * v + 3]));
                        red_add_v4(p.dk_acc + off + 32 * c + 4 * v, __uint_as_float(g[4 * v]) * p.scale,
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

// dq_acc[row] = scale * sum_i dS'_i kd_i over the row's own depth entries (a
// plain store that initialises the accumulator; zero when Ld = 0). Four
// threads per query row, each owning 16 feature pairs.
__global__ void __launch_bounds__(256) bwd_depth_dq_kernel(BwdArgs a) {
    const FwdArgs& f = a.f;
    constexpr int TPR = 4, NP = kD / (2 * TPR);
    const long long rows = (long long)f.B * f.T * f.Hq;
    const long long row = (long long)blockIdx.x * (blockDim.x / TPR) + threadIdx.x / TPR;
    const int u = threadIdx.x % TPR;
    const bool valid = row < rows;
    const long long rc = valid ? row : rows - 1;
    const int h = rc % f.Hq;
    const int t = (rc / f.Hq) % f.T;
    const int b = rc / ((long long)f.Hq * f.T);
    const int kvh = h / f.G;
    const __nv_bfloat16* Q = static_cast<const __nv_bfloat16*>(f.q) + rc * kD;
    const __nv_bfloat16* DO = static_cast<const __nv_bfloat16*>(a.dout) + rc * kD;
    float2 q[NP], dO[NP], acc[NP];
#pragma unroll
    for (int i = 0; i < NP; ++i) {
        const int c = 2 * (TPR * i + u);
        q[i] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(Q + c));
        dO[i] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(DO + c));
        acc[i] = make_float2(0.f, 0.f);
    }
    const long long rix = ((long long)b * f.Hq + h) * f.T + t;
    const float lse2 = f.lse[rix] * kLog2e, Drow = a.rowD[rix], sl2 = f.scale * kLog2e;
    for (int i = 0; i < f.Ld; ++i) {
        const long long off = ((((long long)b * f.T + t) * f.Ld + i) * f.Hkv + kvh) * kD;
        const __nv_bfloat16* KD = static_cast<const __nv_bfloat16*>(f.kd) + off;
        const __nv_bfloat16* VD = static_cast<const __nv_bfloat16*>(f.vd) + off;
        float2 kr[NP];
        float s = 0.f, dp = 0.f;
#pragma unroll
        for (int e = 0; e < NP; ++e) {
            const int c = 2 * (TPR * e + u);
            kr[e] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(KD + c));
            const float2 vr = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(VD + c));
            s = fmaf(q[e].x, kr[e].x, fmaf(q[e].y, kr[e].y, s));
            dp = fmaf(dO[e].x, vr.x, fmaf(dO[e].y, vr.y, dp));
        }
#pragma unroll
        for (int o = 1; o < TPR; o <<= 1) {
            s += __shfl_xor_sync(0xffffffffu, s, o);
            dp += __shfl_xor_sync(0xffffffffu, dp, o);
        }
        const float ds = exp2f(s * sl2 - lse2) * (dp - Drow);
#pragma unroll
        for (int e = 0; e < NP; ++e) {
            acc[e].x = fmaf(ds, kr[e].x, acc[e].x);
            acc[e].y = fmaf(ds, kr[e].y, acc[e].y);
        }
    }
    if (valid) {
        float* dst = a.dq_acc + rc * kD;
#pragma unroll
        for (int e = 0; e < NP; ++e) {
            const int c = 2 * (TPR * e + u);
            *reinterpret_cast<float2*>(dst + c) = make_float2(acc[e].x * f.scale, acc[e].y * f.scale);
        }
    }
}

// fp32 accumulator -> bf16 (dq, dk, dv).
__global__ void dq_convert_kernel(const float4* acc, uint2* dq, long long n4) {
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
         i += (long long)gridDim.x * blockDim.x) {
        const float4 v = acc[i];
        dq[i] = make_uint2(ptx::pack_bf16x2(v.x, v.y), ptx::pack_bf16x2(v.z, v.w));
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
    if (!a.dq_acc) return false;
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
    cudaError_t e = launch_bwd_rowdot(a, s);
    if (e != cudaSuccess) return e;
    {
        const long long rows = (long long)f.B * f.T * f.Hq;
        bwd_depth_dq_kernel<<<(unsigned)((rows + 63) / 64), 256, 0, s>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if ((e = launch_bwd_depth_dkv(a, s)) != cudaSuccess) return e;

    TcBwdParams p;
    memset(&p, 0, sizeof(p));
    const int G = f.G, n = 128 / G;
    const cuuint64_t es = 2;
    {
        const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)f.Hq, (cuuint64_t)f.T, (cuuint64_t)f.B};
        const cuuint64_t st[3] = {kD * es, (cuuint64_t)f.Hq * kD * es, (cuuint64_t)f.T * f.Hq * kD * es};
        const cuuint32_t box[4] = {64, (cuuint32_t)G, (cuuint32_t)n, 1};
        if (!make_tmap_bf16_4d(&p.tm_q, f.q, dims, st, box)) return cudaErrorInvalidValue;
        if (!make_tmap_bf16_4d(&p.tm_do, a.dout, dims, st, box)) return cudaErrorInvalidValue;
    }
    {
        const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)f.Hkv, (cuuint64_t)f.T, (cuuint64_t)f.B};
        const cuuint64_t st[3] = {kD * es, (cuuint64_t)f.Hkv * kD * es, (cuuint64_t)f.T * f.Hkv * kD * es};
        const cuuint32_t box[4] = {64, 1, (cuuint32_t)kBK, 1};
        if (!make_tmap_bf16_4d(&p.tm_k, f.k, dims, st, box)) return cudaErrorInvalidValue;
        if (!make_tmap_bf16_4d(&p.tm_v, f.v, dims, st, box)) return cudaErrorInvalidValue;
    }
    p.lse = f.lse;
    p.rowD = a.rowD;
    p.dq_acc = a.dq_acc;
    p.dk_acc = a.dk_acc;
    p.dv_acc = a.dv_acc;
    p.B = f.B; p.T = f.T; p.Hq = f.Hq; p.Hkv = f.Hkv; p.G = G; p.n = n;
    p.nkt = (f.T + kBK - 1) / kBK;
    // Query tiles per CTA: enough CTAs for ~4 waves over the SMs, at least
    // 16 tiles each so the dK / dV flush stays small against the work.
    {
        long long steps = 0;
        for (int kt = 0; kt < p.nkt; ++kt) steps += (f.T - kt * kBK + n - 1) / n;
        steps *= (long long)f.B * f.Hkv;
        long long qc = (steps + 4LL * sm_count() - 1) / (4LL * sm_count());
        if (qc < 16) qc = 16;
        p.qchunk = (int)qc;
    }
    p.sl2 = f.scale * kLog2e;
    p.scale = f.scale;
    p.status = f.status;
    p.wait_limit = f.wait_limit;
    if ((e = cudaFuncSetAttribute(moda_bwd_seq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  kSmemBytes)) != cudaSuccess)
        return e;
    const size_t kv_bytes = (size_t)f.B * f.T * f.Hkv * kD * sizeof(float);
    if ((e = cudaMemsetAsync(a.dk_acc, 0, kv_bytes, s)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(a.dv_acc, 0, kv_bytes, s)) != cudaSuccess) return e;
    const int n_chunks = ((f.T + n - 1) / n + p.qchunk - 1) / p.qchunk;
    dim3 grid(p.nkt, n_chunks, f.B * f.Hkv);
    moda_bwd_seq_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    auto convert = [&](const float* acc, void* dst, long long elems) {
        const long long n4 = elems / 4;
        long long blocks = (n4 + 255) / 256;
        if (blocks > (long long)sm_count() * 8) blocks = (long long)sm_count() * 8;
        dq_convert_kernel<<<(unsigned)blocks, 256, 0, s>>>(reinterpret_cast<const float4*>(acc),
                                                           static_cast<uint2*>(dst), n4);
        return cudaGetLastError();
    };
    if ((e = convert(a.dq_acc, a.dq, (long long)f.B * f.T * f.Hq * kD)) != cudaSuccess) return e;
    if ((e = convert(a.dk_acc, a.dk, (long long)f.B * f.T * f.Hkv * kD)) != cudaSuccess) return e;
    return convert(a.dv_acc, a.dv, (long long)f.B * f.T * f.Hkv * kD);
}

}  // namespace moda
