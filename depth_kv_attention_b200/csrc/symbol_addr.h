// Device addresses of the library's file-scope __device__ variables, cached
// per device and keyed on the identity of the CUDA context they were
// resolved in.
//
// In host code the name of a __device__ variable denotes a host-side stand-in;
// kernels need the variable's device address, which cudaGetSymbolAddress
// returns for the context current on the calling thread. That address is only
// valid in that context: after cudaDeviceReset (or once the primary context
// has been released and created again) the module loads at a new address. So
// each cache entry remembers the context's unique id (cuCtxGetId) and is
// resolved again when the current context's id differs. The lookup takes a
// mutex, so concurrent first calls from several host threads are safe.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

namespace moda {

class SymbolAddr {
  public:
    explicit SymbolAddr(const void* symbol) : symbol_(symbol) {}

    // Device address of the symbol in the current context of the current
    // device. Outside the first call per context this is two driver queries
    // and a locked table lookup; cudaGetSymbolAddress (which may load the
    // module, and so should not first run inside a stream capture) is called
    // only when the context is new.
    cudaError_t get(void** out) {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
        unsigned long long id = 0;
        const bool have_id = context_id(&id);
        std::lock_guard<std::mutex> lock(mu_);
        Entry& en = table_[dev];
        if (en.addr && have_id && en.ctx_id == id) {
            *out = en.addr;
            return cudaSuccess;
        }
        void* a = nullptr;
        e = cudaGetSymbolAddress(&a, symbol_);
        if (e != cudaSuccess) return e;
        // the context exists now even if it did not before the call
        unsigned long long id2 = 0;
        const bool have_id2 = context_id(&id2);
        en.addr = a;
        en.ctx_id = have_id2 ? id2 : 0;
        *out = a;
        return cudaSuccess;
    }

  private:
    static constexpr int kMaxDevices = 64;
    struct Entry {
        void* addr = nullptr;
        unsigned long long ctx_id = 0;
    };

    typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
    typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

    // Unique id of the calling thread's current context; false when there is
    // none yet or the driver does not offer the query (then every call
    // resolves the address again, which is correct, only slower).
    static bool context_id(unsigned long long* id) {
        static CtxGetCurrentFn get_current = nullptr;
        static CtxGetIdFn get_id = nullptr;
        static std::once_flag once;
        std::call_once(once, [] {
            void* f = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
                q == cudaDriverEntryPointSuccess)
                get_current = reinterpret_cast<CtxGetCurrentFn>(f);
            f = nullptr;
            if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
                q == cudaDriverEntryPointSuccess)
                get_id = reinterpret_cast<CtxGetIdFn>(f);
        });
        if (!get_current || !get_id) return false;
        CUcontext ctx = nullptr;
        if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
        return get_id(ctx, id) == CUDA_SUCCESS;
    }

    const void* symbol_;
    std::mutex mu_;
    Entry table_[kMaxDevices];
};

}  // namespace moda
