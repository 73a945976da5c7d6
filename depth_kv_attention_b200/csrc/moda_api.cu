// Host side of the C ABI declared in include/moda.h: argument validation,
// kernel-family selection and launch. No device allocation and no
// synchronisation (except moda_device_status, and moda_fwd_host's own
// streams and events), no state beyond the device status word and the test
// hook's wait limit.
#include <atomic>
#include <cstdint>
#include <cstring>

#include "moda_internal.h"
#include "symbol_addr.h"

namespace moda {

// One word per device that a kernel sets when a bounded wait expires. It is
// a file-scope __device__ variable, so the library itself never allocates.
__device__ unsigned int g_status_word;

namespace {

constexpr int kMaxDevices = 64;
SymbolAddr g_status_addr(&g_status_word);
std::atomic<unsigned int> g_wait_limit[kMaxDevices];

// Device address of the status word in the current context (resolved per
// context, see symbol_addr.h) and the wait limit set for this device.
cudaError_t status_ptr(unsigned int** p, unsigned int* wait_limit) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    void* a = nullptr;
    e = g_status_addr.get(&a);
    if (e != cudaSuccess) return e;
    *p = static_cast<unsigned int*>(a);
    if (wait_limit) *wait_limit = g_wait_limit[dev].load(std::memory_order_relaxed);
    return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

moda_status check_dims(int B, int T, int Hq, int Hkv, int d, int Ld) {
    if (B < 1 || T < 1 || Hq < 1 || Hkv < 1 || d < 1 || Ld < 0) return MODA_ERR_INVALID_VALUE;
    if (Hq % Hkv) return MODA_ERR_INVALID_VALUE;
    if (d > 128) return MODA_ERR_UNSUPPORTED;
    // Row offsets are formed in 64-bit; the grid uses T and Hq in 32-bit dims.
    if ((long long)B * T * Hq > (1LL << 40)) return MODA_ERR_UNSUPPORTED;
    return MODA_OK;
}

moda_status fill_fwd(FwdArgs& a, const void* q, const void* k, const void* v, const void* kd,
                     const void* vd, int B, int T, int Hq, int Hkv, int d, int Ld, moda_dtype dt,
                     float scale, void* out, float* lse, bool packed) {
    moda_status st = check_dims(B, T, Hq, Hkv, d, Ld);
    if (st != MODA_OK) return st;
    if (dt != MODA_BF16 && dt != MODA_F32) return MODA_ERR_INVALID_VALUE;
    if (!q || !k || !v || !out) return MODA_ERR_INVALID_VALUE;
    if (Ld > 0 && (!kd || !vd)) return MODA_ERR_INVALID_VALUE;
    if (!(scale == scale)) return MODA_ERR_INVALID_VALUE;  // NaN scale
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse) ||
        (Ld > 0 && (!aligned16(kd) || !aligned16(vd))))
        return MODA_ERR_MISALIGNED;
    std::memset(&a, 0, sizeof(a));
    a.q = q; a.k = k; a.v = v; a.kd = kd; a.vd = vd; a.out = out; a.lse = lse;
    a.B = B; a.T = T; a.Hq = Hq; a.Hkv = Hkv; a.G = Hq / Hkv; a.d = d; a.Ld = Ld;
    a.scale = scale;
    a.sq = strides_q(T, Hq, d);
    a.so = a.sq;
    a.skv = strides_q(T, Hkv, d);
    a.sdep = packed ? strides_depth_packed(T, Ld, Hkv, d) : strides_depth_native(T, Ld, Hkv, d);
    a.dtype = dt;
    return MODA_OK;
}

// Depth-slot masks: 8-byte aligned, one 64-bit word per token, so Ld <= 64.
moda_status set_sel(FwdArgs& a, const uint64_t* depth_sel) {
    if (!depth_sel) return MODA_OK;
    if ((reinterpret_cast<uintptr_t>(depth_sel) & 7u) != 0) return MODA_ERR_MISALIGNED;
    if (a.Ld > 64) return MODA_ERR_UNSUPPORTED;
    a.depth_sel = reinterpret_cast<const unsigned long long*>(depth_sel);
    return MODA_OK;
}

moda_status run_fwd(FwdArgs& a, void* stream, moda_impl impl) {
    cudaError_t e = status_ptr(&a.status, &a.wait_limit);
    if (e != cudaSuccess) return MODA_ERR_CUDA;
    const bool tc_ok = fwd_tc_supported(a);
    if ((impl == MODA_IMPL_TC || impl == MODA_IMPL_TC2) && !tc_ok) return MODA_ERR_UNSUPPORTED;
    if (impl == MODA_IMPL_TC2 && !fwd_pair_supported(a)) return MODA_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // a query-token range is a tensor-core forward option only
    if ((a.q_tok0 || a.q_tok1) && (!tc_ok || impl == MODA_IMPL_SIMT || impl == MODA_IMPL_TC2))
        return MODA_ERR_UNSUPPORTED;
    if (impl == MODA_IMPL_SIMT || (impl == MODA_IMPL_AUTO && !tc_ok)) e = launch_fwd_simt(a, s);
    else if (impl == MODA_IMPL_TC2) e = launch_fwd_pair(a, s);
    else e = launch_fwd_tc(a, s);
    return e == cudaSuccess ? MODA_OK : MODA_ERR_LAUNCH;
}

// Workspace: [fp32 D, B*Hq*T, rounded to 256 B] then, for bf16 (tensor-core
// path), the fp32 accumulators of dk and dv [B,T,Hkv,d].
size_t bwd_ws_rowD_bytes(int B, int T, int Hq) {
    return ((size_t)B * Hq * T * sizeof(float) + 255) & ~size_t(255);
}
size_t bwd_ws_bytes(int B, int T, int Hq, int Hkv, int d, bool with_acc) {
    size_t acc = with_acc ? (size_t)B * T * 2 * Hkv * d * sizeof(float) : 0;
    return bwd_ws_rowD_bytes(B, T, Hq) + acc;
}

// Staging layout of moda_fwd_host: q, k, v, kd, vd, out, lse, each at a
// 256-byte-aligned offset. Returns the total size; offs[] receives offsets.
size_t host_staging_layout(int B, int T, int Hq, int Hkv, int d, int Ld, moda_dtype dt, size_t offs[7]) {
    const size_t esz = dt == MODA_F32 ? 4 : 2;
    const size_t n[7] = {(size_t)B * T * Hq * d * esz, (size_t)B * T * Hkv * d * esz,
                         (size_t)B * T * Hkv * d * esz, (size_t)B * T * Ld * Hkv * d * esz,
                         (size_t)B * T * Ld * Hkv * d * esz, (size_t)B * T * Hq * d * esz,
                         (size_t)B * Hq * T * sizeof(float)};
    size_t o = 0;
    for (int i = 0; i < 7; ++i) {
        offs[i] = o;
        o += (n[i] + 255) & ~size_t(255);
    }
    return o;
}

}  // namespace
}  // namespace moda

using namespace moda;

extern "C" {

int moda_abi_version(void) { return MODA_ABI_VERSION; }

const char* moda_status_string(moda_status s) {
    switch (s) {
        case MODA_OK: return "MODA_OK";
        case MODA_ERR_INVALID_VALUE: return "MODA_ERR_INVALID_VALUE";
        case MODA_ERR_UNSUPPORTED: return "MODA_ERR_UNSUPPORTED";
        case MODA_ERR_MISALIGNED: return "MODA_ERR_MISALIGNED";
        case MODA_ERR_WORKSPACE: return "MODA_ERR_WORKSPACE";
        case MODA_ERR_LAUNCH: return "MODA_ERR_LAUNCH";
        case MODA_ERR_DEVICE_TIMEOUT: return "MODA_ERR_DEVICE_TIMEOUT";
        case MODA_ERR_CUDA: return "MODA_ERR_CUDA";
    }
    return "MODA_ERR_UNKNOWN";
}

moda_status moda_fwd_sel(const void* q, const void* k, const void* v, const void* kd,
                         const void* vd, const uint64_t* depth_sel, int B, int T, int Hq, int Hkv,
                         int d, int Ld, moda_dtype dtype, float scale, void* out, float* lse,
                         void* stream, moda_impl impl) {
    if (impl != MODA_IMPL_AUTO && impl != MODA_IMPL_SIMT && impl != MODA_IMPL_TC && impl != MODA_IMPL_TC2)
        return MODA_ERR_INVALID_VALUE;
    FwdArgs a;
    moda_status st = fill_fwd(a, q, k, v, kd, vd, B, T, Hq, Hkv, d, Ld, dtype, scale, out, lse, false);
    if (st != MODA_OK) return st;
    st = set_sel(a, depth_sel);
    if (st != MODA_OK) return st;
    return run_fwd(a, stream, impl);
}

moda_status moda_fwd_ex(const void* q, const void* k, const void* v, const void* kd, const void* vd,
                        int B, int T, int Hq, int Hkv, int d, int Ld, moda_dtype dtype, float scale,
                        void* out, float* lse, void* stream, moda_impl impl) {
    return moda_fwd_sel(q, k, v, kd, vd, nullptr, B, T, Hq, Hkv, d, Ld, dtype, scale, out, lse,
                        stream, impl);
}

moda_status moda_fwd(const void* q, const void* k, const void* v, const void* kd, const void* vd,
                     int B, int T, int Hq, int Hkv, int d, int Ld, moda_dtype dtype, float scale,
                     void* out, float* lse, void* stream) {
    return moda_fwd_ex(q, k, v, kd, vd, B, T, Hq, Hkv, d, Ld, dtype, scale, out, lse, stream,
                       MODA_IMPL_AUTO);
}

size_t moda_bwd_workspace_bytes(int B, int T, int Hq, int Hkv, int d, int Ld, moda_dtype dtype) {
    if (check_dims(B, T, Hq, Hkv, d, Ld) != MODA_OK) return 0;
    if (dtype != MODA_BF16 && dtype != MODA_F32) return 0;
    // The fp32 accumulators are reserved for every bf16 shape so that the
    // size does not depend on which kernel family a call selects.
    return bwd_ws_bytes(B, T, Hq, Hkv, d, dtype == MODA_BF16);
}

moda_status moda_bwd_sel(const void* q, const void* k, const void* v, const void* kd,
                         const void* vd, const uint64_t* depth_sel, const void* out,
                         const float* lse, const void* dout, int B, int T, int Hq, int Hkv, int d,
                         int Ld, moda_dtype dtype, float scale, void* dq, void* dk, void* dv,
                         void* dkd, void* dvd, void* workspace, size_t workspace_bytes,
                         void* stream, moda_impl impl) {
    if (impl != MODA_IMPL_AUTO && impl != MODA_IMPL_SIMT && impl != MODA_IMPL_TC && impl != MODA_IMPL_TC2)
        return MODA_ERR_INVALID_VALUE;
    BwdArgs a;
    std::memset(&a, 0, sizeof(a));
    moda_status st = fill_fwd(a.f, q, k, v, kd, vd, B, T, Hq, Hkv, d, Ld, dtype, scale,
                              const_cast<void*>(out), const_cast<float*>(lse), false);
    if (st != MODA_OK) return st;
    st = set_sel(a.f, depth_sel);
    if (st != MODA_OK) return st;
    if (!lse || !dout || !dq || !dk || !dv) return MODA_ERR_INVALID_VALUE;
    if (Ld > 0 && (!dkd || !dvd)) return MODA_ERR_INVALID_VALUE;
    if (!aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
        (Ld > 0 && (!aligned16(dkd) || !aligned16(dvd))))
        return MODA_ERR_MISALIGNED;
    const size_t need = moda_bwd_workspace_bytes(B, T, Hq, Hkv, d, Ld, dtype);
    if (!workspace || workspace_bytes < need) return MODA_ERR_WORKSPACE;
    if (!aligned16(workspace)) return MODA_ERR_MISALIGNED;
    a.dout = dout; a.dq = dq; a.dk = dk; a.dv = dv; a.dkd = dkd; a.dvd = dvd;
    a.rowD = static_cast<float*>(workspace);
    if (dtype == MODA_BF16) {
        char* base = static_cast<char*>(workspace) + bwd_ws_rowD_bytes(B, T, Hq);
        a.dk_acc = reinterpret_cast<float*>(base);
        a.dv_acc = a.dk_acc + (size_t)B * T * Hkv * d;
    }
    cudaError_t e = status_ptr(&a.f.status, &a.f.wait_limit);
    if (e != cudaSuccess) return MODA_ERR_CUDA;
    const bool tc_ok = bwd_tc_supported(a);
    if ((impl == MODA_IMPL_TC || impl == MODA_IMPL_TC2) && !tc_ok) return MODA_ERR_UNSUPPORTED;
    const bool use_tc = impl == MODA_IMPL_TC || impl == MODA_IMPL_TC2 || (impl == MODA_IMPL_AUTO && tc_ok);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    e = use_tc ? launch_bwd_tc(a, s) : launch_bwd_simt(a, s);
    return e == cudaSuccess ? MODA_OK : MODA_ERR_LAUNCH;
}

moda_status moda_bwd_ex(const void* q, const void* k, const void* v, const void* kd, const void* vd,
                        const void* out, const float* lse, const void* dout, int B, int T, int Hq,
                        int Hkv, int d, int Ld, moda_dtype dtype, float scale, void* dq, void* dk,
                        void* dv, void* dkd, void* dvd, void* workspace, size_t workspace_bytes,
                        void* stream, moda_impl impl) {
    return moda_bwd_sel(q, k, v, kd, vd, nullptr, out, lse, dout, B, T, Hq, Hkv, d, Ld, dtype,
                        scale, dq, dk, dv, dkd, dvd, workspace, workspace_bytes, stream, impl);
}

moda_status moda_bwd(const void* q, const void* k, const void* v, const void* kd, const void* vd,
                     const void* out, const float* lse, const void* dout, int B, int T, int Hq,
                     int Hkv, int d, int Ld, moda_dtype dtype, float scale, void* dq, void* dk,
                     void* dv, void* dkd, void* dvd, void* workspace, size_t workspace_bytes,
                     void* stream) {
    return moda_bwd_ex(q, k, v, kd, vd, out, lse, dout, B, T, Hq, Hkv, d, Ld, dtype, scale, dq, dk,
                       dv, dkd, dvd, workspace, workspace_bytes, stream, MODA_IMPL_AUTO);
}

size_t moda_pack_depth_bytes(int B, int T, int Hkv, int d, int Ld, moda_dtype dtype) {
    if (B < 1 || T < 1 || Hkv < 1 || d < 1 || d > 128 || Ld < 0) return 0;
    if (dtype != MODA_BF16 && dtype != MODA_F32) return 0;
    const size_t esz = dtype == MODA_F32 ? 4 : 2;
    return 2 * (size_t)B * T * Ld * Hkv * d * esz;
}

moda_status moda_pack_depth(const void* kd, const void* vd, int B, int T, int Hkv, int d, int Ld,
                            moda_dtype dtype, void* packed, void* stream) {
    if (B < 1 || T < 1 || Hkv < 1 || d < 1 || Ld < 0) return MODA_ERR_INVALID_VALUE;
    if (dtype != MODA_BF16 && dtype != MODA_F32) return MODA_ERR_INVALID_VALUE;
    if (d > 128) return MODA_ERR_UNSUPPORTED;
    if (Ld == 0) return MODA_OK;
    if (!kd || !vd || !packed) return MODA_ERR_INVALID_VALUE;
    if (!aligned16(kd) || !aligned16(vd) || !aligned16(packed)) return MODA_ERR_MISALIGNED;
    const int esz = dtype == MODA_F32 ? 4 : 2;
    if ((d * esz) % 16) return MODA_ERR_UNSUPPORTED;  // 16-byte vector copies
    cudaError_t e = launch_pack_depth(kd, vd, B, T, Hkv, d, Ld, dtype, packed,
                                      static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MODA_OK : MODA_ERR_LAUNCH;
}

moda_status moda_depth_write(const void* k, const void* v, int B, int T, int Hkv, int d, int Ld,
                             int slot, moda_dtype dtype, void* kd, void* vd, void* stream) {
    if (B < 1 || T < 1 || Hkv < 1 || d < 1 || Ld < 1) return MODA_ERR_INVALID_VALUE;
    if (slot < 0 || slot >= Ld) return MODA_ERR_INVALID_VALUE;
    if (dtype != MODA_BF16 && dtype != MODA_F32) return MODA_ERR_INVALID_VALUE;
    if (!k || !v || !kd || !vd) return MODA_ERR_INVALID_VALUE;
    if (!aligned16(k) || !aligned16(v) || !aligned16(kd) || !aligned16(vd)) return MODA_ERR_MISALIGNED;
    const int esz = dtype == MODA_F32 ? 4 : 2;
    if ((d * esz) % 16) return MODA_ERR_UNSUPPORTED;  // 16-byte vector copies
    if ((long long)B * T * Ld * Hkv * d >= (1LL << 48)) return MODA_ERR_UNSUPPORTED;
    cudaError_t e = launch_depth_write(k, v, B, T, Hkv, d, Ld, slot, dtype, kd, vd,
                                       static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MODA_OK : MODA_ERR_LAUNCH;
}

moda_status moda_fwd_q8(const void* q, const void* k, const void* v, const int8_t* kd8, const int8_t* vd8,
                        const float* kd_scale, const float* vd_scale, int B, int T, int Hq, int Hkv, int d,
                        int Ld, moda_dtype dtype, float scale, void* out, float* lse, void* stream,
                        moda_impl impl) {
    if (impl != MODA_IMPL_AUTO && impl != MODA_IMPL_SIMT && impl != MODA_IMPL_TC && impl != MODA_IMPL_TC2)
        return MODA_ERR_INVALID_VALUE;
    FwdArgs a;
    moda_status st = fill_fwd(a, q, k, v, kd8, vd8, B, T, Hq, Hkv, d, Ld, dtype, scale, out, lse, false);
    if (st != MODA_OK) return st;
    if (Ld > 0) {
        if (!kd_scale || !vd_scale) return MODA_ERR_INVALID_VALUE;
        if ((reinterpret_cast<uintptr_t>(kd_scale) & 3u) || (reinterpret_cast<uintptr_t>(vd_scale) & 3u))
            return MODA_ERR_MISALIGNED;
        a.depth_q8 = 1;
        a.kd_scale = kd_scale;
        a.vd_scale = vd_scale;
    }
    return run_fwd(a, stream, impl);
}

namespace {
moda_status check_q8_out(const int8_t* kd8, const int8_t* vd8, const float* ks, const float* vs) {
    if (!kd8 || !vd8 || !ks || !vs) return MODA_ERR_INVALID_VALUE;
    if ((reinterpret_cast<uintptr_t>(ks) & 3u) || (reinterpret_cast<uintptr_t>(vs) & 3u)) return MODA_ERR_MISALIGNED;
    return MODA_OK;
}
}  // namespace

moda_status moda_depth_quantize_q8(const void* kd, const void* vd, int B, int T, int Hkv, int d, int Ld,
                                   moda_dtype dtype, int8_t* kd8, int8_t* vd8, float* kd_scale,
                                   float* vd_scale, void* stream) {
    if (B < 1 || T < 1 || Hkv < 1 || d < 1 || Ld < 0) return MODA_ERR_INVALID_VALUE;
    if (dtype != MODA_BF16 && dtype != MODA_F32) return MODA_ERR_INVALID_VALUE;
    if (d > 128) return MODA_ERR_UNSUPPORTED;
    if (Ld == 0) return MODA_OK;
    if (!kd || !vd) return MODA_ERR_INVALID_VALUE;
    moda_status st = check_q8_out(kd8, vd8, kd_scale, vd_scale);
    if (st != MODA_OK) return st;
    const long long rows = (long long)B * T * Ld * Hkv;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = launch_quantize_q8(kd, rows, d, dtype, 1, 1, 0, kd8, kd_scale, s);
    if (e == cudaSuccess) e = launch_quantize_q8(vd, rows, d, dtype, 1, 1, 0, vd8, vd_scale, s);
    return e == cudaSuccess ? MODA_OK : MODA_ERR_LAUNCH;
}

moda_status moda_depth_write_q8(const void* k, const void* v, int B, int T, int Hkv, int d, int Ld, int slot,
                                moda_dtype dtype, int8_t* kd8, int8_t* vd8, float* kd_scale, float* vd_scale,
                                void* stream) {
    if (B < 1 || T < 1 || Hkv < 1 || d < 1 || Ld < 1) return MODA_ERR_INVALID_VALUE;
    if (slot < 0 || slot >= Ld) return MODA_ERR_INVALID_VALUE;
    if (dtype != MODA_BF16 && dtype != MODA_F32) return MODA_ERR_INVALID_VALUE;
    if (d > 128) return MODA_ERR_UNSUPPORTED;
    if (!k || !v) return MODA_ERR_INVALID_VALUE;
    moda_status st = check_q8_out(kd8, vd8, kd_scale, vd_scale);
    if (st != MODA_OK) return st;
    // input row (b, t, h) -> depth row ((b*T + t)*Ld + slot)*Hkv + h
    const long long rows = (long long)B * T * Hkv;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = launch_quantize_q8(k, rows, d, dtype, Hkv, (long long)Ld * Hkv, (long long)slot * Hkv, kd8,
                                       kd_scale, s);
    if (e == cudaSuccess)
        e = launch_quantize_q8(v, rows, d, dtype, Hkv, (long long)Ld * Hkv, (long long)slot * Hkv, vd8, vd_scale, s);
    return e == cudaSuccess ? MODA_OK : MODA_ERR_LAUNCH;
}

moda_status moda_depth_slot_layout(int B, int T, int Hkv, int d, int Ld, int slot, long long* offset,
                                   long long strides[4]) {
    if (B < 1 || T < 1 || Hkv < 1 || d < 1 || Ld < 1 || slot < 0 || slot >= Ld) return MODA_ERR_INVALID_VALUE;
    if (!offset || !strides) return MODA_ERR_INVALID_VALUE;
    const Strides5 sd = strides_depth_native(T, Ld, Hkv, d);
    *offset = (long long)slot * sd.si;
    strides[0] = sd.sb;
    strides[1] = sd.st;
    strides[2] = sd.sh;
    strides[3] = 1;
    return MODA_OK;
}

moda_status moda_fwd_packed(const void* q, const void* k, const void* v, const void* packed_depth,
                            int B, int T, int Hq, int Hkv, int d, int Ld, moda_dtype dtype,
                            float scale, void* out, float* lse, void* stream) {
    const size_t half = moda_pack_depth_bytes(B, T, Hkv, d, Ld, dtype) / 2;
    const void* kd = packed_depth;
    const void* vd = packed_depth ? static_cast<const char*>(packed_depth) + half : nullptr;
    FwdArgs a;
    moda_status st = fill_fwd(a, q, k, v, kd, vd, B, T, Hq, Hkv, d, Ld, dtype, scale, out, lse, true);
    if (st != MODA_OK) return st;
    return run_fwd(a, stream, MODA_IMPL_AUTO);
}

size_t moda_fwd_host_staging_bytes(int B, int T, int Hq, int Hkv, int d, int Ld, moda_dtype dtype) {
    if (check_dims(B, T, Hq, Hkv, d, Ld) != MODA_OK) return 0;
    if (dtype != MODA_BF16 && dtype != MODA_F32) return 0;
    size_t offs[7];
    return host_staging_layout(B, T, Hq, Hkv, d, Ld, dtype, offs);
}

namespace {

// RAII holder of the extra streams and events of the pipelined host forward.
struct HostPipe {
    cudaStream_t sc = nullptr, so = nullptr;
    cudaEvent_t ev[2 * 64 + 1] = {};
    int n_ev = 0;
    ~HostPipe() {
        for (int i = 0; i < n_ev; ++i) cudaEventDestroy(ev[i]);  // released once recorded work completes
        if (sc) cudaStreamDestroy(sc);
        if (so) cudaStreamDestroy(so);
    }
    cudaEvent_t event() {
        cudaEvent_t e = nullptr;
        if (n_ev >= (int)(sizeof(ev) / sizeof(ev[0])) ||
            cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess)
            return nullptr;
        ev[n_ev++] = e;
        return e;
    }
};

// Token rows [t0, t1) of every batch of a [B, T, row_bytes] tensor, host <-> device:
// one 2D copy (B rows of (t1 - t0) * row_bytes, pitch T * row_bytes), or a
// plain copy when the range is the whole tensor.
bool copy_rows(void* dst, const void* src, int B, int T, size_t row_bytes, int t0, int t1, cudaMemcpyKind kind,
               cudaStream_t s) {
    if (row_bytes == 0 || t1 <= t0) return true;
    const size_t off = (size_t)t0 * row_bytes, width = (size_t)(t1 - t0) * row_bytes, pitch = (size_t)T * row_bytes;
    char* d = static_cast<char*>(dst) + off;
    const char* h = static_cast<const char*>(src) + off;
    if (B == 1 || width == pitch) return cudaMemcpyAsync(d, h, width * B, kind, s) == cudaSuccess;
    return cudaMemcpy2DAsync(d, pitch, h, pitch, width, (size_t)B, kind, s) == cudaSuccess;
}

}  // namespace

moda_status moda_fwd_host(const void* q, const void* k, const void* v, const void* kd, const void* vd,
                          int B, int T, int Hq, int Hkv, int d, int Ld, moda_dtype dtype, float scale,
                          void* out, float* lse, void* staging, size_t staging_bytes, void* stream) {
    moda_status st = check_dims(B, T, Hq, Hkv, d, Ld);
    if (st != MODA_OK) return st;
    if (dtype != MODA_BF16 && dtype != MODA_F32) return MODA_ERR_INVALID_VALUE;
    if (!q || !k || !v || !out) return MODA_ERR_INVALID_VALUE;
    if (Ld > 0 && (!kd || !vd)) return MODA_ERR_INVALID_VALUE;
    size_t offs[7];
    const size_t need = host_staging_layout(B, T, Hq, Hkv, d, Ld, dtype, offs);
    if (!staging || staging_bytes < need) return MODA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(staging) & 255u) != 0) return MODA_ERR_MISALIGNED;
    char* base = static_cast<char*>(staging);
    void* dq = base + offs[0];
    void* dk = base + offs[1];
    void* dv = base + offs[2];
    void* dkd = Ld > 0 ? base + offs[3] : nullptr;
    void* dvd = Ld > 0 ? base + offs[4] : nullptr;
    void* dout = base + offs[5];
    float* dlse = lse ? reinterpret_cast<float*>(base + offs[6]) : nullptr;
    const size_t esz = dtype == MODA_F32 ? 4 : 2;
    const size_t rq = (size_t)Hq * d * esz, rkv = (size_t)Hkv * d * esz, rdep = (size_t)Ld * Hkv * d * esz;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    FwdArgs a;
    st = fill_fwd(a, dq, dk, dv, dkd, dvd, B, T, Hq, Hkv, d, Ld, dtype, scale, dout, dlse, false);
    if (st != MODA_OK) return st;
    const int unit = fwd_tc_supported(a) ? fwd_tc_unit_tokens(a) : 0;
    const int nblk = unit ? (T + unit - 1) / unit : 0;
    if (nblk < 2) {
        // one pass: inputs to the device, the forward, outputs back
        const void* src[5] = {q, k, v, kd, vd};
        void* dst[5] = {dq, dk, dv, dkd, dvd};
        const size_t rb[5] = {rq, rkv, rkv, rdep, rdep};
        for (int i = 0; i < 5; ++i)
            if (!copy_rows(dst[i], src[i], B, T, rb[i], 0, T, cudaMemcpyHostToDevice, s)) return MODA_ERR_CUDA;
        st = run_fwd(a, stream, MODA_IMPL_AUTO);
        if (st != MODA_OK) return st;
        if (!copy_rows(out, dout, B, T, rq, 0, T, cudaMemcpyDeviceToHost, s)) return MODA_ERR_CUDA;
        if (lse && cudaMemcpyAsync(lse, dlse, (size_t)B * Hq * T * sizeof(float), cudaMemcpyDeviceToHost, s) !=
                       cudaSuccess)
            return MODA_ERR_CUDA;
        return MODA_OK;
    }
    // Pipelined over chunks of query tokens (whole work units): the caller's
    // stream copies chunk j's rows of q, k, v, kd, vd; an internal stream runs
    // the forward of chunk j's queries once they are in (causal: they need
    // the keys of chunks 0..j only, copied before them on the same stream);
    // a second internal stream copies chunk j's output rows back while the
    // next chunks are copied and computed. The caller's stream waits for all
    // of it at the end. A chunk's last key tile (128 keys) and last depth
    // chunk (128 depth rows) reach past its last token: those keys are masked
    // (P = 0), but 0 * NaN from a row not yet copied would still reach O, so
    // each chunk also copies the keys up to 128 tokens and the depth rows up
    // to 128 rows ahead (every row once: the copies continue where the last
    // one ended).
    HostPipe hp;
    if (cudaStreamCreateWithFlags(&hp.sc, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&hp.so, cudaStreamNonBlocking) != cudaSuccess)
        return MODA_ERR_CUDA;
    // An error after work went onto the internal streams still orders the
    // caller's stream after that work (or, if that cannot be enqueued, waits
    // for it here), so the caller may release its buffers once its own stream
    // is done.
    auto fail = [&](moda_status e) {
        cudaStream_t inner[2] = {hp.sc, hp.so};
        for (cudaStream_t t : inner) {
            cudaEvent_t j = nullptr;
            const bool joined = cudaEventCreateWithFlags(&j, cudaEventDisableTiming) == cudaSuccess &&
                                cudaEventRecord(j, t) == cudaSuccess && cudaStreamWaitEvent(s, j, 0) == cudaSuccess;
            if (j) cudaEventDestroy(j);
            if (!joined) cudaStreamSynchronize(t);
        }
        return e;
    };
    const int nch = nblk < 16 ? nblk : 16;
    const int ahead_kv = 128, ahead_dep = Ld > 0 ? (128 + Ld - 1) / Ld : 0;
    int kv_end = 0, dep_end = 0;  // tokens copied so far of k, v and of kd, vd
    for (int j = 0; j < nch; ++j) {
        const int t0 = (int)((long long)nblk * j / nch) * unit;
        const int t1 = j + 1 == nch ? T : (int)((long long)nblk * (j + 1) / nch) * unit;
        const int kv_to = t1 + ahead_kv < T ? t1 + ahead_kv : T;
        const int dep_to = t1 + ahead_dep < T ? t1 + ahead_dep : T;
        if (!copy_rows(dq, q, B, T, rq, t0, t1, cudaMemcpyHostToDevice, s) ||
            !copy_rows(dk, k, B, T, rkv, kv_end, kv_to, cudaMemcpyHostToDevice, s) ||
            !copy_rows(dv, v, B, T, rkv, kv_end, kv_to, cudaMemcpyHostToDevice, s) ||
            !copy_rows(dkd, kd, B, T, rdep, dep_end, dep_to, cudaMemcpyHostToDevice, s) ||
            !copy_rows(dvd, vd, B, T, rdep, dep_end, dep_to, cudaMemcpyHostToDevice, s))
            return fail(MODA_ERR_CUDA);
        kv_end = kv_to;
        dep_end = dep_to;
        cudaEvent_t in = hp.event(), done = hp.event();
        if (!in || !done) return fail(MODA_ERR_CUDA);
        if (cudaEventRecord(in, s) != cudaSuccess || cudaStreamWaitEvent(hp.sc, in, 0) != cudaSuccess)
            return fail(MODA_ERR_CUDA);
        a.q_tok0 = t0;
        a.q_tok1 = t1;
        st = run_fwd(a, hp.sc, MODA_IMPL_TC);
        if (st != MODA_OK) return fail(st);
        if (cudaEventRecord(done, hp.sc) != cudaSuccess || cudaStreamWaitEvent(hp.so, done, 0) != cudaSuccess)
            return fail(MODA_ERR_CUDA);
        if (!copy_rows(out, dout, B, T, rq, t0, t1, cudaMemcpyDeviceToHost, hp.so)) return fail(MODA_ERR_CUDA);
    }
    // the so stream already waits for the last chunk's forward, hence for all
    if (lse && cudaMemcpyAsync(lse, dlse, (size_t)B * Hq * T * sizeof(float), cudaMemcpyDeviceToHost, hp.so) !=
                   cudaSuccess)
        return fail(MODA_ERR_CUDA);
    cudaEvent_t fin = hp.event();
    if (!fin || cudaEventRecord(fin, hp.so) != cudaSuccess || cudaStreamWaitEvent(s, fin, 0) != cudaSuccess)
        return fail(MODA_ERR_CUDA);
    return MODA_OK;
}

moda_status moda_device_status(void* stream) {
    unsigned int* p = nullptr;
    if (status_ptr(&p, nullptr) != cudaSuccess) return MODA_ERR_CUDA;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MODA_ERR_CUDA;
    unsigned int w = 0;
    if (cudaMemcpy(&w, p, sizeof(w), cudaMemcpyDeviceToHost) != cudaSuccess) return MODA_ERR_CUDA;
    if (w) {
        const unsigned int zero = 0;
        if (cudaMemcpy(p, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
            return MODA_ERR_CUDA;
        return MODA_ERR_DEVICE_TIMEOUT;
    }
    return MODA_OK;
}

moda_status moda_debug_exp2_poly(const float* x, float* y, int n, void* stream) {
    if (n < 0 || (n > 0 && (!x || !y))) return MODA_ERR_INVALID_VALUE;
    if (n == 0) return MODA_OK;
    cudaError_t e = launch_exp2_poly(x, y, n, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MODA_OK : MODA_ERR_LAUNCH;
}

moda_status moda_debug_set_wait_limit(uint32_t spins) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MODA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return MODA_ERR_CUDA;
    g_wait_limit[dev].store(spins, std::memory_order_relaxed);
    return MODA_OK;
}

}  // extern "C"
