// Scalar (SIMT, fp32 FMA) MoDA kernels: forward, backward and the depth repack.
//
// These run any shape the ABI accepts (d <= 128, any G, fp32 or bf16) and are
// the path for fp32 inputs. The arithmetic is the MoDA read step: one online
// softmax over the same-token depth keys and the causal sequence keys
// ("动态混合深度注意力机制MoDA技术解析", mhpn.cn, §1.2 formula; §2.2 online softmax
// state m / acc / o and the dual mask).
//
// Thread layout: TPR threads cooperate on one query row (or one key row in the
// dK/dV kernel). Thread u of the group owns the feature pairs
// {2*(TPR*i + u), 2*(TPR*i + u) + 1}, so that the group reads contiguous
// 8*TPR-byte chunks of a shared-memory row and partial dot products combine
// with log2(TPR) xor-shuffles.
#include <cuda_bf16.h>

#include <cmath>

#include "moda_internal.h"

namespace moda {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kDMax = 128;
constexpr int kKT = 32;  // keys per shared-memory tile

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <>
__device__ __forceinline__ float to_f<int8_t>(int8_t x) { return (float)x; }

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Feature pairs owned by one of TPR threads: NP = kDMax / (2 * TPR).
template <int TPR>
struct Split {
    static constexpr int NP = kDMax / (2 * TPR);
    __device__ static __forceinline__ int feat(int i, int u) { return 2 * (TPR * i + u); }
};

template <int TPR>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
    for (int o = 1; o < TPR; o <<= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Load the feature pairs this thread owns from a global row (zero past d).
template <int TPR, typename T>
__device__ __forceinline__ void load_row(const T* row, int d, int u, float2 (&r)[Split<TPR>::NP],
                                         float mul = 1.f) {
#pragma unroll
    for (int i = 0; i < Split<TPR>::NP; ++i) {
        const int c = Split<TPR>::feat(i, u);
        r[i].x = (c < d) ? to_f(row[c]) * mul : 0.f;
        r[i].y = (c + 1 < d) ? to_f(row[c + 1]) * mul : 0.f;
    }
}

// 8-bit depth row: fl32(scale * code), then rounded to the input dtype T
// (the type the unquantised depth cache would hold).
template <int TPR, typename T>
__device__ __forceinline__ void load_row_q8(const int8_t* row, int d, int u, float2 (&r)[Split<TPR>::NP],
                                            float sigma) {
    load_row<TPR>(row, d, u, r, sigma);
#pragma unroll
    for (int i = 0; i < Split<TPR>::NP; ++i) {
        r[i].x = to_f(from_f<T>(r[i].x));
        r[i].y = to_f(from_f<T>(r[i].y));
    }
}

template <int TPR, typename T>
__device__ __forceinline__ void store_row(T* row, int d, int u, const float2 (&r)[Split<TPR>::NP],
                                          float mul) {
#pragma unroll
    for (int i = 0; i < Split<TPR>::NP; ++i) {
        const int c = Split<TPR>::feat(i, u);
        if (c < d) row[c] = from_f<T>(r[i].x * mul);
        if (c + 1 < d) row[c + 1] = from_f<T>(r[i].y * mul);
    }
}

template <int TPR>
__device__ __forceinline__ float dot_smem(const float2 (&a)[Split<TPR>::NP], const float* srow, int u) {
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < Split<TPR>::NP; ++i) {
        const float2 b = *reinterpret_cast<const float2*>(srow + Split<TPR>::feat(i, u));
        s = fmaf(a[i].x, b.x, s);
        s = fmaf(a[i].y, b.y, s);
    }
    return s;
}

template <int TPR>
__device__ __forceinline__ float dot_regs(const float2 (&a)[Split<TPR>::NP], const float2 (&b)[Split<TPR>::NP]) {
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < Split<TPR>::NP; ++i) {
        s = fmaf(a[i].x, b[i].x, s);
        s = fmaf(a[i].y, b[i].y, s);
    }
    return s;
}

template <int TPR>
__device__ __forceinline__ void axpy_smem(float2 (&acc)[Split<TPR>::NP], float p, const float* srow, int u) {
#pragma unroll
    for (int i = 0; i < Split<TPR>::NP; ++i) {
        const float2 b = *reinterpret_cast<const float2*>(srow + Split<TPR>::feat(i, u));
        acc[i].x = fmaf(p, b.x, acc[i].x);
        acc[i].y = fmaf(p, b.y, acc[i].y);
    }
}

template <int TPR>
__device__ __forceinline__ void axpy_regs(float2 (&acc)[Split<TPR>::NP], float p, const float2 (&b)[Split<TPR>::NP]) {
#pragma unroll
    for (int i = 0; i < Split<TPR>::NP; ++i) {
        acc[i].x = fmaf(p, b[i].x, acc[i].x);
        acc[i].y = fmaf(p, b[i].y, acc[i].y);
    }
}

// Stage rows [r0, r0 + n) of a [*, d] slice (row stride `rs` elements) into a
// zero-padded fp32 shared tile of kDMax columns.
template <typename T>
__device__ __forceinline__ void stage_rows(float* s, const T* base, long long rs, int r0, int n,
                                           int nmax, int d) {
    for (int e = threadIdx.x; e < nmax * kDMax; e += blockDim.x) {
        const int r = e / kDMax, c = e % kDMax;
        s[e] = (r < n && c < d) ? to_f(base[(long long)(r0 + r) * rs + c]) : 0.f;
    }
}

// ---------------------------------------------------------------- forward
// CTA = (token block of n_tok tokens) x (head block of hpc heads of one kv
// group), one row per (token, head), token-major: row = tok * hpc + head.
template <typename T>
__global__ void __launch_bounds__(128) fwd_simt_kernel(FwdArgs a, int n_tok, int hpc) {
    constexpr int TPR = 2;
    using S = Split<TPR>;
    __shared__ __align__(16) float sK[kKT * kDMax];
    __shared__ __align__(16) float sV[kKT * kDMax];

    const int hblocks = (a.G + hpc - 1) / hpc;
    const int kvh = blockIdx.y / hblocks, hb = blockIdx.y % hblocks, b = blockIdx.z;
    const int t0 = (gridDim.x - 1 - blockIdx.x) * n_tok;  // heaviest (latest) tokens first
    const int row = threadIdx.x / TPR, u = threadIdx.x % TPR;
    const int tl = row / hpc, gl = row % hpc;
    const int t = t0 + tl, g = hb * hpc + gl;
    const bool valid = tl < n_tok && t < a.T && g < a.G;
    const int tc = min(t, a.T - 1), gc = min(g, a.G - 1);
    const int h = kvh * a.G + gc;
    const T* Q = static_cast<const T*>(a.q);
    const T* K = static_cast<const T*>(a.k);
    const T* V = static_cast<const T*>(a.v);
    const T* KD = static_cast<const T*>(a.kd);
    const T* VD = static_cast<const T*>(a.vd);

    float2 q[S::NP], o[S::NP];
    const float qmul = a.scale * kLog2e;  // logits in the log2 domain
    load_row<TPR>(Q + b * a.sq.sb + tc * a.sq.st + h * a.sq.sh, a.d, u, q, qmul);
#pragma unroll
    for (int i = 0; i < S::NP; ++i) o[i] = make_float2(0.f, 0.f);
    float m = -INFINITY, l = 0.f;

    // Depth keys of the same token (depth mask), of the slots the token
    // selects: read straight from global. Rows of one warp select different
    // slots, so every lane runs the shuffles of group_sum and an unselected
    // slot is skipped only after them.
    const unsigned long long sel = a.depth_sel ? a.depth_sel[(long long)b * a.T + tc] : 0ull;
    for (int i = 0; i < a.Ld; ++i) {
        const long long off = b * a.sdep.sb + tc * a.sdep.st + (long long)i * a.sdep.si + kvh * a.sdep.sh;
        float2 kr[S::NP];
        const long long srow = off / a.d;  // (b, t, i, kvh) row of the 8-bit scales
        if (a.depth_q8)
            load_row_q8<TPR, T>(static_cast<const int8_t*>(a.kd) + off, a.d, u, kr, a.kd_scale[srow]);
        else
            load_row<TPR>(KD + off, a.d, u, kr);
        const float s = group_sum<TPR>(dot_regs<TPR>(q, kr));
        if (a.depth_sel && !((sel >> i) & 1ull)) continue;
        float2 vr[S::NP];
        if (a.depth_q8)
            load_row_q8<TPR, T>(static_cast<const int8_t*>(a.vd) + off, a.d, u, vr, a.vd_scale[srow]);
        else
            load_row<TPR>(VD + off, a.d, u, vr);
        if (s > m) {
            const float corr = exp2f(m - s);
            l *= corr;
#pragma unroll
            for (int c = 0; c < S::NP; ++c) { o[c].x *= corr; o[c].y *= corr; }
            m = s;
        }
        const float p = exp2f(s - m);
        l += p;
        axpy_regs<TPR>(o, p, vr);
    }

    // Causal sequence keys 0..t.
    const int t_last = min(a.T, t0 + n_tok) - 1;
    const T* Kb = K + b * a.skv.sb + kvh * a.skv.sh;
    const T* Vb = V + b * a.skv.sb + kvh * a.skv.sh;
    for (int j0 = 0; j0 <= t_last; j0 += kKT) {
        const int n = min(kKT, t_last - j0 + 1);
        __syncthreads();
        stage_rows(sK, Kb, a.skv.st, j0, n, kKT, a.d);
        stage_rows(sV, Vb, a.skv.st, j0, n, kKT, a.d);
        __syncthreads();
        for (int jj = 0; jj < n; ++jj) {
            const float s = group_sum<TPR>(dot_smem<TPR>(q, sK + jj * kDMax, u));
            if (j0 + jj <= t) {
                if (s > m) {
                    const float corr = exp2f(m - s);
                    l *= corr;
#pragma unroll
                    for (int c = 0; c < S::NP; ++c) { o[c].x *= corr; o[c].y *= corr; }
                    m = s;
                }
                const float p = exp2f(s - m);
                l += p;
                axpy_smem<TPR>(o, p, sV + jj * kDMax, u);
            }
        }
    }

    if (valid) {
        T* O = static_cast<T*>(a.out);
        store_row<TPR>(O + b * a.so.sb + t * a.so.st + h * a.so.sh, a.d, u, o, 1.f / l);
        if (a.lse && u == 0) a.lse[((long long)b * a.Hq + h) * a.T + t] = m * kLn2 + logf(l);
    }
}

// --------------------------------------------------------------- backward
// D[b,h,t] = <dout, out>: one warp per row.
template <typename T>
__global__ void bwd_rowdot_kernel(BwdArgs a) {
    const long long rows = (long long)a.f.B * a.f.T * a.f.Hq;
    const long long r = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    if (r >= rows) return;
    const int lane = threadIdx.x % 32;
    const int h = r % a.f.Hq;
    const int t = (r / a.f.Hq) % a.f.T;
    const int b = r / ((long long)a.f.Hq * a.f.T);
    const T* O = static_cast<const T*>(a.f.out) + b * a.f.so.sb + t * a.f.so.st + h * a.f.so.sh;
    const T* dO = static_cast<const T*>(a.dout) + b * a.f.so.sb + t * a.f.so.st + h * a.f.so.sh;
    float s = 0.f;
    for (int c = lane; c < a.f.d; c += 32) s = fmaf(to_f(O[c]), to_f(dO[c]), s);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) a.rowD[((long long)b * a.f.Hq + h) * a.f.T + t] = s;
}

// dq for every query row: causal keys and same-token depth keys.
// The row statistic D = sum_j P_j dP_j: rowD holds the estimate
// D~ = <dout, out> on entry (out as the forward stored it); the row's pass
// over all its keys accumulates delta = sum_j P_j (dP_j - D~) (= D - D~, as
// sum_j P_j = 1) and bq = sum_j P_j k_j, writes dq = scale (sum_j P_j (dP_j -
// D~) k_j - delta bq) and stores D = D~ + delta for the dK/dV kernels.
template <typename T>
__global__ void __launch_bounds__(256) bwd_dq_simt_kernel(BwdArgs a, int n_tok, int hpc) {
    constexpr int TPR = 4;
    using S = Split<TPR>;
    __shared__ __align__(16) float sK[kKT * kDMax];
    __shared__ __align__(16) float sV[kKT * kDMax];
    const FwdArgs& f = a.f;
    const int hblocks = (f.G + hpc - 1) / hpc;
    const int kvh = blockIdx.y / hblocks, hb = blockIdx.y % hblocks, b = blockIdx.z;
    const int t0 = (gridDim.x - 1 - blockIdx.x) * n_tok;
    const int row = threadIdx.x / TPR, u = threadIdx.x % TPR;
    const int tl = row / hpc, gl = row % hpc;
    const int t = t0 + tl, g = hb * hpc + gl;
    const bool valid = tl < n_tok && t < f.T && g < f.G;
    const int tc = min(t, f.T - 1), gc = min(g, f.G - 1);
    const int h = kvh * f.G + gc;

    float2 q[S::NP], dO[S::NP], dq[S::NP], bq[S::NP];
    load_row<TPR>(static_cast<const T*>(f.q) + b * f.sq.sb + tc * f.sq.st + h * f.sq.sh, f.d, u, q,
                  f.scale * kLog2e);
    load_row<TPR>(static_cast<const T*>(a.dout) + b * f.so.sb + tc * f.so.st + h * f.so.sh, f.d, u, dO);
#pragma unroll
    for (int i = 0; i < S::NP; ++i) {
        dq[i] = make_float2(0.f, 0.f);
        bq[i] = make_float2(0.f, 0.f);
    }
    const long long rix = ((long long)b * f.Hq + h) * f.T + tc;
    const float lse2 = f.lse[rix] * kLog2e;
    const float Drow = a.rowD[rix];
    float delta = 0.f;

    // Depth part: dq += dS'_i kd_i over the selected slots (skipped only
    // after the warp-wide shuffles of group_sum, as in the forward).
    const unsigned long long sel = f.depth_sel ? f.depth_sel[(long long)b * f.T + tc] : 0ull;
    for (int i = 0; i < f.Ld; ++i) {
        const long long off = b * f.sdep.sb + tc * f.sdep.st + (long long)i * f.sdep.si + kvh * f.sdep.sh;
        float2 kr[S::NP], vr[S::NP];
        load_row<TPR>(static_cast<const T*>(f.kd) + off, f.d, u, kr);
        load_row<TPR>(static_cast<const T*>(f.vd) + off, f.d, u, vr);
        const float s = group_sum<TPR>(dot_regs<TPR>(q, kr));
        const float dp = group_sum<TPR>(dot_regs<TPR>(dO, vr));
        if (f.depth_sel && !((sel >> i) & 1ull)) continue;
        const float p = exp2f(s - lse2);
        const float ds = p * (dp - Drow);
        delta += ds;
        axpy_regs<TPR>(dq, ds, kr);
        axpy_regs<TPR>(bq, p, kr);
    }
    const int t_last = min(f.T, t0 + n_tok) - 1;
    const T* Kb = static_cast<const T*>(f.k) + b * f.skv.sb + kvh * f.skv.sh;
    const T* Vb = static_cast<const T*>(f.v) + b * f.skv.sb + kvh * f.skv.sh;
    for (int j0 = 0; j0 <= t_last; j0 += kKT) {
        const int n = min(kKT, t_last - j0 + 1);
        __syncthreads();
        stage_rows(sK, Kb, f.skv.st, j0, n, kKT, f.d);
        stage_rows(sV, Vb, f.skv.st, j0, n, kKT, f.d);
        __syncthreads();
        for (int jj = 0; jj < n; ++jj) {
            const float s = group_sum<TPR>(dot_smem<TPR>(q, sK + jj * kDMax, u));
            const float dp = group_sum<TPR>(dot_smem<TPR>(dO, sV + jj * kDMax, u));
            if (j0 + jj <= t) {
                const float p = exp2f(s - lse2);
                const float ds = p * (dp - Drow);
                delta += ds;
                axpy_smem<TPR>(dq, ds, sK + jj * kDMax, u);
                axpy_smem<TPR>(bq, p, sK + jj * kDMax, u);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < S::NP; ++i) {
        dq[i].x = fmaf(-delta, bq[i].x, dq[i].x);
        dq[i].y = fmaf(-delta, bq[i].y, dq[i].y);
    }
    if (valid) {
        store_row<TPR>(static_cast<T*>(a.dq) + b * f.sq.sb + t * f.sq.st + h * f.sq.sh, f.d, u, dq, f.scale);
        if (u == 0) a.rowD[rix] = Drow + delta;
    }
}

// dk, dv for every sequence key j: rows t >= j of the G heads of its group.
template <typename T>
__global__ void __launch_bounds__(256) bwd_dkv_simt_kernel(BwdArgs a, int n_key) {
    constexpr int TPR = 4;
    using S = Split<TPR>;
    constexpr int kRT = 16;  // query rows staged per shared tile
    __shared__ __align__(16) float sQ[kRT * kDMax];
    __shared__ __align__(16) float sdO[kRT * kDMax];
    __shared__ float sL[kRT], sD[kRT];
    const FwdArgs& f = a.f;
    const int kvh = blockIdx.y, b = blockIdx.z;
    const int j0 = blockIdx.x * n_key;
    const int kr = threadIdx.x / TPR, u = threadIdx.x % TPR;
    const int j = j0 + kr;
    const bool valid = kr < n_key && j < f.T;
    const int jc = min(j, f.T - 1);

    float2 k[S::NP], v[S::NP], dk[S::NP], dv[S::NP];
    const long long kvoff = b * f.skv.sb + jc * f.skv.st + kvh * f.skv.sh;
    load_row<TPR>(static_cast<const T*>(f.k) + kvoff, f.d, u, k, f.scale * kLog2e);
    load_row<TPR>(static_cast<const T*>(f.v) + kvoff, f.d, u, v);
#pragma unroll
    for (int i = 0; i < S::NP; ++i) { dk[i] = make_float2(0.f, 0.f); dv[i] = make_float2(0.f, 0.f); }

    // Query rows in token-major order (t, g) for t >= j0 of this group.
    const long long nrows = (long long)(f.T - j0) * f.G;
    for (long long r0 = 0; r0 < nrows; r0 += kRT) {
        const int n = (int)(nrows - r0 < kRT ? nrows - r0 : kRT);
        __syncthreads();
        for (int e = threadIdx.x; e < kRT * kDMax; e += blockDim.x) {
            const int r = e / kDMax, c = e % kDMax;
            float qv = 0.f, dov = 0.f;
            if (r < n && c < f.d) {
                const long long rr = r0 + r;
                const int t = j0 + (int)(rr / f.G), h = kvh * f.G + (int)(rr % f.G);
                qv = to_f(static_cast<const T*>(f.q)[b * f.sq.sb + t * f.sq.st + h * f.sq.sh + c]);
                dov = to_f(static_cast<const T*>(a.dout)[b * f.so.sb + t * f.so.st + h * f.so.sh + c]);
            }
            sQ[e] = qv;
            sdO[e] = dov;
        }
        for (int r = threadIdx.x; r < kRT; r += blockDim.x) {
            float L = 0.f, D = 0.f;
            if (r < n) {
                const long long rr = r0 + r;
                const int t = j0 + (int)(rr / f.G), h = kvh * f.G + (int)(rr % f.G);
                const long long rix = ((long long)b * f.Hq + h) * f.T + t;
                L = f.lse[rix] * kLog2e;
                D = a.rowD[rix];
            }
            sL[r] = L;
            sD[r] = D;
        }
        __syncthreads();
        for (int r = 0; r < n; ++r) {
            const int t = j0 + (int)((r0 + r) / f.G);
            const float s = group_sum<TPR>(dot_smem<TPR>(k, sQ + r * kDMax, u));
            const float dp = group_sum<TPR>(dot_smem<TPR>(v, sdO + r * kDMax, u));
            if (t >= j) {
                const float p = exp2f(s - sL[r]);
                axpy_smem<TPR>(dv, p, sdO + r * kDMax, u);
                axpy_smem<TPR>(dk, p * (dp - sD[r]), sQ + r * kDMax, u);
            }
        }
    }
    if (valid) {
        store_row<TPR>(static_cast<T*>(a.dk) + kvoff, f.d, u, dk, f.scale);
        store_row<TPR>(static_cast<T*>(a.dv) + kvoff, f.d, u, dv, 1.f);
    }
}

// dkd, dvd: one TPR-group per (b, t, i, kvh); sums over the G heads of token t.
template <typename T>
__global__ void __launch_bounds__(256) bwd_depth_simt_kernel(BwdArgs a) {
    constexpr int TPR = 4;
    using S = Split<TPR>;
    const FwdArgs& f = a.f;
    const long long items = (long long)f.B * f.T * f.Ld * f.Hkv;
    const long long it = (long long)blockIdx.x * (blockDim.x / TPR) + threadIdx.x / TPR;
    const int u = threadIdx.x % TPR;
    const bool valid = it < items;
    const long long itc = valid ? it : items - 1;
    const int kvh = itc % f.Hkv;
    const int i = (itc / f.Hkv) % f.Ld;
    const int t = (itc / ((long long)f.Hkv * f.Ld)) % f.T;
    const int b = itc / ((long long)f.Hkv * f.Ld * f.T);
    const long long off = b * f.sdep.sb + t * f.sdep.st + (long long)i * f.sdep.si + kvh * f.sdep.sh;
    float2 kd[S::NP], vd[S::NP], dkd[S::NP], dvd[S::NP];
    load_row<TPR>(static_cast<const T*>(f.kd) + off, f.d, u, kd, f.scale * kLog2e);
    load_row<TPR>(static_cast<const T*>(f.vd) + off, f.d, u, vd);
#pragma unroll
    for (int c = 0; c < S::NP; ++c) { dkd[c] = make_float2(0.f, 0.f); dvd[c] = make_float2(0.f, 0.f); }
    // An unselected slot is absent from every row: zero gradients (its
    // probabilities are zeroed; the loop itself stays warp-uniform because
    // group_sum shuffles across the whole warp).
    const bool selected = !f.depth_sel || ((f.depth_sel[(long long)b * f.T + t] >> i) & 1ull);
    for (int g = 0; g < f.G; ++g) {
        const int h = kvh * f.G + g;
        float2 q[S::NP], dO[S::NP];
        load_row<TPR>(static_cast<const T*>(f.q) + b * f.sq.sb + t * f.sq.st + h * f.sq.sh, f.d, u, q);
        load_row<TPR>(static_cast<const T*>(a.dout) + b * f.so.sb + t * f.so.st + h * f.so.sh, f.d, u, dO);
        const long long rix = ((long long)b * f.Hq + h) * f.T + t;
        const float s = group_sum<TPR>(dot_regs<TPR>(q, kd));
        const float dp = group_sum<TPR>(dot_regs<TPR>(dO, vd));
        const float p = selected ? exp2f(s - f.lse[rix] * kLog2e) : 0.f;
        axpy_regs<TPR>(dvd, p, dO);
        axpy_regs<TPR>(dkd, p * (dp - a.rowD[rix]), q);
    }
    if (valid) {
        store_row<TPR>(static_cast<T*>(a.dkd) + off, f.d, u, dkd, f.scale);
        store_row<TPR>(static_cast<T*>(a.dvd) + off, f.d, u, dvd, 1.f);
    }
}

// ------------------------------------------------------------ depth repack
// [B,T,Ld,Hkv,d] -> [B,Hkv,T*Ld,d] for kd then vd, 16-byte vectors.
__global__ void pack_depth_kernel(const uint4* kd, const uint4* vd, uint4* out, int B, int T,
                                  int Hkv, int Ld, int vec_per_row) {
    const long long per = (long long)B * T * Ld * Hkv * vec_per_row;
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < 2 * per;
         e += (long long)gridDim.x * blockDim.x) {
        const int which = e >= per;
        const long long x = e - which * per;  // index in source order
        const int c = x % vec_per_row;
        const int h = (x / vec_per_row) % Hkv;
        const long long ti = (x / ((long long)vec_per_row * Hkv)) % ((long long)T * Ld);
        const int b = x / ((long long)vec_per_row * Hkv * T * Ld);
        const long long dst = (((long long)b * Hkv + h) * T * Ld + ti) * vec_per_row + c;
        out[which * per + dst] = (which ? vd : kd)[x];
    }
}

void simt_tiling(int G, int rows_target, int& n_tok, int& hpc) {
    hpc = G < rows_target ? G : rows_target;
    n_tok = rows_target / hpc;
    if (n_tok < 1) n_tok = 1;
}

}  // namespace

cudaError_t launch_fwd_simt(const FwdArgs& a, cudaStream_t s) {
    int n_tok, hpc;
    simt_tiling(a.G, 64, n_tok, hpc);
    dim3 grid((a.T + n_tok - 1) / n_tok, a.Hkv * ((a.G + hpc - 1) / hpc), a.B);
    if (a.dtype == MODA_F32)
        fwd_simt_kernel<float><<<grid, 128, 0, s>>>(a, n_tok, hpc);
    else
        fwd_simt_kernel<__nv_bfloat16><<<grid, 128, 0, s>>>(a, n_tok, hpc);
    return cudaGetLastError();
}

cudaError_t launch_bwd_simt(const BwdArgs& a, cudaStream_t s) {
    const FwdArgs& f = a.f;
    const long long rows = (long long)f.B * f.T * f.Hq;
    const bool f32 = f.dtype == MODA_F32;
    {
        dim3 grid((unsigned)((rows + 7) / 8));
        if (f32) bwd_rowdot_kernel<float><<<grid, 256, 0, s>>>(a);
        else bwd_rowdot_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(a);
    }
    {
        int n_tok, hpc;
        simt_tiling(f.G, 64, n_tok, hpc);
        dim3 grid((f.T + n_tok - 1) / n_tok, f.Hkv * ((f.G + hpc - 1) / hpc), f.B);
        if (f32) bwd_dq_simt_kernel<float><<<grid, 256, 0, s>>>(a, n_tok, hpc);
        else bwd_dq_simt_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(a, n_tok, hpc);
    }
    {
        const int n_key = 64;
        dim3 grid((f.T + n_key - 1) / n_key, f.Hkv, f.B);
        if (f32) bwd_dkv_simt_kernel<float><<<grid, 256, 0, s>>>(a, n_key);
        else bwd_dkv_simt_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(a, n_key);
    }
    if (f.Ld > 0) {
        const long long items = (long long)f.B * f.T * f.Ld * f.Hkv;
        dim3 grid((unsigned)((items + 63) / 64));
        if (f32) bwd_depth_simt_kernel<float><<<grid, 256, 0, s>>>(a);
        else bwd_depth_simt_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(a);
    }
    return cudaGetLastError();
}

// The write step: k / v [B,T,Hkv,d] into slot `slot` of kd / vd
// [B,T,Ld,Hkv,d], 16-byte vectors. One (b, t) row of k is Hkv*vec vectors
// and lands contiguously at kd[b, t, slot], so both sides stay coalesced.
__global__ void depth_write_kernel(const uint4* k, const uint4* v, uint4* kd, uint4* vd, long long rows,
                                   int row_vec, int Ld, int slot) {
    const long long per = rows * row_vec;
    for (long long x = (long long)blockIdx.x * blockDim.x + threadIdx.x; x < 2 * per;
         x += (long long)gridDim.x * blockDim.x) {
        const bool is_v = x >= per;
        const long long y = is_v ? x - per : x;
        const long long row = y / row_vec;  // b * T + t
        const int c = (int)(y % row_vec);
        const long long dst = (row * Ld + slot) * row_vec + c;
        if (is_v) vd[dst] = v[y];
        else kd[dst] = k[y];
    }
}

cudaError_t launch_depth_write(const void* k, const void* v, int B, int T, int Hkv, int d, int Ld,
                               int slot, moda_dtype dt, void* kd, void* vd, cudaStream_t s) {
    const int esz = dt == MODA_F32 ? 4 : 2;
    const int row_vec = Hkv * (d * esz / 16);
    const long long rows = (long long)B * T;
    const long long total = 2 * rows * row_vec;
    if (total == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    long long blocks = (total + 255) / 256;
    if (blocks > (long long)sms * 8) blocks = (long long)sms * 8;
    depth_write_kernel<<<(unsigned)blocks, 256, 0, s>>>(static_cast<const uint4*>(k), static_cast<const uint4*>(v),
                                                        static_cast<uint4*>(kd), static_cast<uint4*>(vd), rows,
                                                        row_vec, Ld, slot);
    return cudaGetLastError();
}

namespace {
// 8-bit depth KV: one warp per row of d <= 128 values. amax over the row,
// scale = amax / 127 and code = round-half-even(x / scale) clamped to
// [-127, 127], each a single IEEE fp32 operation (__fdiv_rn, __float2int_rn)
// so the codes are exactly those of the float32 definition; an all-zero row
// gets scale 0 and codes 0.
template <typename T>
__global__ void quantize_q8_kernel(const T* x, long long rows, int d, int inner, long long out_tok_stride,
                                   long long out_off, int8_t* codes, float* scales) {
    const long long r = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    if (r >= rows) return;
    const int lane = threadIdx.x % 32;
    const T* row = x + r * d;
    float v[4];
    float amax = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int c = lane + 32 * e;
        v[e] = c < d ? to_f(row[c]) : 0.f;
        amax = fmaxf(amax, fabsf(v[e]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float sigma = __fdiv_rn(amax, 127.f);
    const long long orow = (r / inner) * out_tok_stride + out_off + r % inner;
    int8_t* crow = codes + orow * d;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int c = lane + 32 * e;
        if (c < d) {
            int q = 0;
            if (sigma > 0.f) q = min(127, max(-127, __float2int_rn(__fdiv_rn(v[e], sigma))));
            crow[c] = (int8_t)q;
        }
    }
    if (lane == 0) scales[orow] = sigma;
}
}  // namespace

cudaError_t launch_quantize_q8(const void* x, long long rows, int d, moda_dtype dt, int inner,
                               long long out_tok_stride, long long out_off, int8_t* codes,
                               float* scales, cudaStream_t s) {
    if (rows <= 0) return cudaSuccess;
    const long long blocks = (rows + 7) / 8;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    if (dt == MODA_F32)
        quantize_q8_kernel<float><<<(unsigned)blocks, 256, 0, s>>>(static_cast<const float*>(x), rows, d, inner,
                                                                    out_tok_stride, out_off, codes, scales);
    else
        quantize_q8_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, s>>>(
            static_cast<const __nv_bfloat16*>(x), rows, d, inner, out_tok_stride, out_off, codes, scales);
    return cudaGetLastError();
}

cudaError_t launch_pack_depth(const void* kd, const void* vd, int B, int T, int Hkv, int d, int Ld,
                              moda_dtype dt, void* packed, cudaStream_t s) {
    const int esz = dt == MODA_F32 ? 4 : 2;
    const int vec = d * esz / 16;
    const long long total = 2LL * B * T * Ld * Hkv * vec;
    if (total == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    long long blocks = (total + 255) / 256;
    if (blocks > (long long)sms * 8) blocks = (long long)sms * 8;
    pack_depth_kernel<<<(unsigned)blocks, 256, 0, s>>>(static_cast<const uint4*>(kd),
                                                       static_cast<const uint4*>(vd),
                                                       static_cast<uint4*>(packed), B, T, Hkv, Ld, vec);
    return cudaGetLastError();
}

}  // namespace moda
