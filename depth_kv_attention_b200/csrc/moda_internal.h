// Internal declarations shared by the host ABI (moda_api.cu) and the kernel
// translation units. Not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "../../include/moda.h"

namespace moda {

// Element strides of one tensor family. Every tensor is addressed as
//   base + b*sb + t*st + h*sh (+ i*si for depth tensors) + c   (c = feature).
struct Strides4 {
    long long sb, st, sh;
};
struct Strides5 {
    long long sb, st, si, sh;
};

struct FwdArgs {
    const void* q;
    const void* k;
    const void* v;
    const void* kd;   // may be null when Ld == 0
    const void* vd;
    void* out;
    float* lse;       // may be null
    int B, T, Hq, Hkv, G, d, Ld;
    float scale;
    Strides4 sq, skv, so;
    Strides5 sdep;    // kd and vd share strides
    moda_dtype dtype;
    const unsigned long long* depth_sel;  // [B,T] depth-slot bit masks, or null (all slots)
    // 8-bit depth KV: kd / vd hold int8 codes [B,T,Ld,Hkv,d] and the depth
    // values are scale * code with one fp32 scale per (b,t,i,kvh) row
    int depth_q8;
    const float* kd_scale;    // [B,T,Ld,Hkv]
    const float* vd_scale;
    unsigned int* status;     // device status word
    unsigned int wait_limit;  // bounded-wait polls (0 = kernel default)
    // Query tokens [q_tok0, q_tok1) of this launch (tensor-core forward only;
    // q_tok1 == 0: to T). Keys and depth rows are read from the full tensors,
    // so the keys 0 .. q_tok1-1 must be in place; q_tok0 is a multiple of
    // fwd_tc_unit_tokens().
    int q_tok0, q_tok1;
};

struct BwdArgs {
    FwdArgs f;              // q,k,v,kd,vd, dims, strides; f.out = forward output, f.lse = lse
    const void* dout;       // same layout as q
    void* dq;
    void* dk;
    void* dv;
    void* dkd;
    void* dvd;
    float* rowD;            // [B, Hq, T] fp32 workspace: <dout, out>, then the
                            // dq kernel's exact D = sum_j P_j dP_j
    float* dk_acc;          // [B, T, Hkv, d] fp32 workspace (tensor-core path only)
    float* dv_acc;          // [B, T, Hkv, d] fp32 workspace (tensor-core path only)
};

// Natural layouts of the ABI (packed depth changes sdep only).
inline Strides4 strides_q(int T, int H, int d) {
    return Strides4{(long long)T * H * d, (long long)H * d, (long long)d};
}
inline Strides5 strides_depth_native(int T, int Ld, int Hkv, int d) {
    return Strides5{(long long)T * Ld * Hkv * d, (long long)Ld * Hkv * d,
                    (long long)Hkv * d, (long long)d};
}
inline Strides5 strides_depth_packed(int T, int Ld, int Hkv, int d) {
    return Strides5{(long long)Hkv * T * Ld * d, (long long)Ld * d, (long long)d,
                    (long long)T * Ld * d};
}

// SIMT kernels (moda_simt.cu). Any d <= 128, any G, fp32 or bf16.
cudaError_t launch_fwd_simt(const FwdArgs& a, cudaStream_t s);
cudaError_t launch_bwd_simt(const BwdArgs& a, cudaStream_t s);
cudaError_t launch_pack_depth(const void* kd, const void* vd, int B, int T, int Hkv, int d,
                              int Ld, moda_dtype dt, void* packed, cudaStream_t s);
cudaError_t launch_depth_write(const void* k, const void* v, int B, int T, int Hkv, int d, int Ld,
                               int slot, moda_dtype dt, void* kd, void* vd, cudaStream_t s);
// Per-row int8 quantisation of `rows` rows of d values (input dtype dt):
// input row r -> output row (r / inner) * out_tok_stride + out_off + r % inner
// of codes [*, d] and scales [*].
cudaError_t launch_quantize_q8(const void* x, long long rows, int d, moda_dtype dt, int inner,
                               long long out_tok_stride, long long out_off, int8_t* codes,
                               float* scales, cudaStream_t s);

// Tensor-core kernels for sm_100a (moda_fwd_sm100.cu, moda_bwd_sm100.cu).
bool fwd_tc_supported(const FwdArgs& a);
// Tokens per work unit of the tensor-core forward (two 128-row query tiles).
inline int fwd_tc_unit_tokens(const FwdArgs& a) { return 2 * (128 / a.G); }
cudaError_t launch_fwd_tc(const FwdArgs& a, cudaStream_t s);
// The CTA-pair forward (moda_fwd_pair_sm100.cu): bf16 depth (not 8-bit).
bool fwd_pair_supported(const FwdArgs& a);
cudaError_t launch_fwd_pair(const FwdArgs& a, cudaStream_t s);
bool bwd_tc_supported(const BwdArgs& a);
cudaError_t launch_bwd_tc(const BwdArgs& a, cudaStream_t s);
// The forward's FMA-pipe exp2 applied element-wise (test hook).
cudaError_t launch_exp2_poly(const float* x, float* y, int n, cudaStream_t s);

}  // namespace moda
