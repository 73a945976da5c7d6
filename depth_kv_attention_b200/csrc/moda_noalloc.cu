// moda_bwd_noalloc: the MoDA backward for callers that cannot allocate device
// memory.
//
// Some callers own no allocator for this library to use: a C or C++ host
// program that hands over only its input and output buffers, or a runtime that
// reserves the whole device for its own memory pool, where a cudaMalloc from a
// library would fail once the pool has claimed the memory, or would bypass the
// runtime's accounting. moda_bwd needs a caller-provided workspace; this entry
// point takes its scratch from a fixed array that lives in the library's own
// device image instead, so the caller passes inputs and outputs only.
//
// Cost of that choice: every GPU that loads the library holds
// MODA_NOALLOC_SCRATCH_BYTES of device memory for the array until the process
// exits. Larger problems are rejected (MODA_ERR_WORKSPACE) rather than
// allocated for.
#include <cstring>

#include "moda_internal.h"
#include "symbol_addr.h"

namespace moda {
namespace {

// The scratch: fp32 row statistics D = rowsum(dout * out), [B, Hq, T].
__device__ __align__(256) unsigned char g_bwd_noalloc_scratch[MODA_NOALLOC_SCRATCH_BYTES];

// In host code `g_bwd_noalloc_scratch` names a host-side stand-in, not the
// device array: a kernel given it would fault or silently touch the wrong
// memory. Its device address is resolved with the device current, once per
// device and context (again after a cudaDeviceReset), and cached.
SymbolAddr g_scratch_addr(g_bwd_noalloc_scratch);

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace moda

using namespace moda;

extern "C" moda_status moda_bwd_noalloc(const void* q, const void* k, const void* v, const void* kd,
                                        const void* vd, const void* out, const float* lse,
                                        const void* dout, int B, int T, int Hq, int Hkv, int d,
                                        int Ld, moda_dtype dtype, float scale, void* dq, void* dk,
                                        void* dv, void* dkd, void* dvd, void* stream) {
    // Same argument rules as moda_bwd.
    if (B < 1 || T < 1 || Hq < 1 || Hkv < 1 || d < 1 || Ld < 0 || Hq % Hkv) return MODA_ERR_INVALID_VALUE;
    if (dtype != MODA_BF16 && dtype != MODA_F32) return MODA_ERR_INVALID_VALUE;
    if (d > 128) return MODA_ERR_UNSUPPORTED;
    if (!(scale == scale)) return MODA_ERR_INVALID_VALUE;
    if (!q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv) return MODA_ERR_INVALID_VALUE;
    if (Ld > 0 && (!kd || !vd || !dkd || !dvd)) return MODA_ERR_INVALID_VALUE;
    const void* ptrs[] = {q, k, v, out, lse, dout, dq, dk, dv};
    for (const void* p : ptrs)
        if (!al16(p)) return MODA_ERR_MISALIGNED;
    if (Ld > 0 && (!al16(kd) || !al16(vd) || !al16(dkd) || !al16(dvd))) return MODA_ERR_MISALIGNED;
    // The scratch has a fixed size: reject what does not fit.
    const unsigned long long need = (unsigned long long)B * Hq * T * sizeof(float);
    if (need > MODA_NOALLOC_SCRATCH_BYTES) return MODA_ERR_WORKSPACE;

    void* scratch = nullptr;
    if (g_scratch_addr.get(&scratch) != cudaSuccess) return MODA_ERR_CUDA;

    BwdArgs a;
    memset(&a, 0, sizeof(a));
    FwdArgs& f = a.f;
    f.q = q; f.k = k; f.v = v; f.kd = kd; f.vd = vd;
    f.out = const_cast<void*>(out);
    f.lse = const_cast<float*>(lse);
    f.B = B; f.T = T; f.Hq = Hq; f.Hkv = Hkv; f.G = Hq / Hkv; f.d = d; f.Ld = Ld;
    f.scale = scale;
    f.sq = strides_q(T, Hq, d);
    f.so = f.sq;
    f.skv = strides_q(T, Hkv, d);
    f.sdep = strides_depth_native(T, Ld, Hkv, d);
    f.dtype = dtype;
    a.dout = dout; a.dq = dq; a.dk = dk; a.dv = dv; a.dkd = dkd; a.dvd = dvd;
    // The backward's first kernel writes every D it later reads, so the
    // previous call's contents need no clearing.
    a.rowD = static_cast<float*>(scratch);
    cudaError_t e = launch_bwd_simt(a, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MODA_OK : MODA_ERR_LAUNCH;
}
