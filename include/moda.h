/*
 * moda.h — C ABI of the B200 (sm_100a) Mixture-of-Depths Attention library.
 *
 * The operation (the MoDA "read" step).  For batch b, query head h, position t
 * and kv-head g = h / G (G = Hq / Hkv, contiguous head groups):
 *
 *     s_j  = scale * <q[b,t,h,:], k[b,j,g,:]>        for j = 0..t        (causal)
 *     s'_i = scale * <q[b,t,h,:], kd[b,t,i,g,:]>     for i = 0..Ld-1     (same token)
 *     p    = softmax over the concatenation [s || s']  (ONE normaliser)
 *     out[b,t,h,:] = sum_j p_j v[b,j,g,:] + sum_i p'_i vd[b,t,i,g,:]
 *     lse[b,h,t]   = log(sum_j e^{s_j} + sum_i e^{s'_i})     (natural log)
 *
 * Sources: "动态混合深度注意力机制MoDA技术解析" (mhpn.cn), §1.2 (the MoDA attention
 * formula: one softmax over the concatenated current-layer and earlier-layer
 * logits scaled by 1/sqrt(d)) and §2.2 (online softmax state m / acc / o, and
 * the dual mask: causal over the sequence, same position over depth);
 * "Mixture-of-Depths Attention" (gist.science, German technical summary),
 * §2 "Methodik" (Read-Step, Unified Softmax, flash-compatible / chunk-aware /
 * group-aware layouts).  Ld = 0 is plain causal GQA attention.
 *
 * Conventions shared by every entry point
 *   - Every tensor argument is a DEVICE pointer to a dense, row-major tensor in
 *     the layout stated below, aligned to 16 bytes (moda_fwd_host: host
 *     buffers, see there). The caller owns every buffer; the library never
 *     allocates device memory, frees or synchronises (except in
 *     moda_device_status, and in moda_fwd_host, which creates two streams and
 *     its events for the call and, after an error, may wait for them) and
 *     keeps no per-call state.
 *   - Layouts:  q, out, dout, dq   [B, T, Hq, d]
 *               k, v, dk, dv       [B, T, Hkv, d]
 *               kd, vd, dkd, dvd   [B, T, Ld, Hkv, d]   (depth keys/values of a
 *                                   token's earlier layers, token-contiguous)
 *               lse                [B, Hq, T]  fp32
 *   - dtype: MODA_BF16 (bf16 storage, fp32 accumulation) or MODA_F32 (fp32
 *     storage and arithmetic). Outputs take the input dtype; lse and the
 *     workspace are fp32.
 *   - stream: a cudaStream_t cast to void*; NULL means the legacy default
 *     stream. Every call only ENQUEUES work and returns; results are ready
 *     when the stream reaches them.
 *   - kd and vd may be NULL iff Ld == 0. Outputs must not alias inputs.
 *   - Argument errors return synchronously with nothing launched. A failed
 *     launch returns MODA_ERR_LAUNCH. A kernel whose bounded wait on an
 *     on-chip barrier expires records MODA_ERR_DEVICE_TIMEOUT in a device
 *     status word that moda_device_status reports; such a kernel skips its
 *     remaining work and returns instead of hanging.
 *   - Supported shapes: B, T, Hq, Hkv >= 1, Hq % Hkv == 0, Ld >= 0,
 *     1 <= d <= 128 for MODA_F32.  MODA_BF16 on the tensor-core path needs
 *     d == 128 and 128 % G == 0; other bf16 shapes run on the SIMT path
 *     (d <= 128). Anything else returns MODA_ERR_UNSUPPORTED.
 *   - Thread safety: entry points may be called concurrently from several
 *     host threads on different streams.
 */
#ifndef MODA_H_
#define MODA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MODA_ABI_VERSION 3

typedef enum {
    MODA_OK = 0,
    MODA_ERR_INVALID_VALUE = 1,   /* NULL pointer, non-positive size, Hq % Hkv != 0 */
    MODA_ERR_UNSUPPORTED = 2,     /* valid shape the library does not implement     */
    MODA_ERR_MISALIGNED = 3,      /* a tensor pointer is not 16-byte aligned         */
    MODA_ERR_WORKSPACE = 4,       /* workspace NULL or smaller than required         */
    MODA_ERR_LAUNCH = 5,          /* the CUDA launch (or tensor-map encode) failed   */
    MODA_ERR_DEVICE_TIMEOUT = 6,  /* a kernel's bounded wait expired (device word)   */
    MODA_ERR_CUDA = 7             /* another CUDA runtime error (device query, sync) */
} moda_status;

typedef enum { MODA_BF16 = 0, MODA_F32 = 1 } moda_dtype;

/* Kernel family selector for moda_fwd_ex / moda_bwd_ex.  AUTO picks the
 * tensor-core path when the shape supports it, else SIMT. MODA_IMPL_TC2 runs
 * the forward on CTA pairs (one M = 256 MMA drives two SMs; bf16 depth only,
 * else MODA_ERR_UNSUPPORTED): the same results, slower than the single-CTA
 * forward that TC and AUTO use on this hardware, kept as a selectable
 * variant. The backward has one tensor-core form, which TC and TC2 select. */
typedef enum { MODA_IMPL_AUTO = 0, MODA_IMPL_SIMT = 1, MODA_IMPL_TC = 2, MODA_IMPL_TC2 = 3 } moda_impl;

/* Version of this ABI (MODA_ABI_VERSION of the library). */
int moda_abi_version(void);

/* Human-readable name of a status code. Never NULL; static storage. */
const char* moda_status_string(moda_status s);

/*
 * moda_fwd — fused MoDA forward: causal sequence attention and same-token
 * depth attention under one online softmax (mhpn.cn §1.2 formula, §2.2 online
 * softmax and dual mask).
 *   q    [B,T,Hq,d]        in   queries
 *   k, v [B,T,Hkv,d]       in   current-layer sequence keys / values
 *   kd, vd [B,T,Ld,Hkv,d]  in   depth keys / values (NULL iff Ld == 0)
 *   scale                  in   logit scale, normally 1/sqrt(d); applied to
 *                               sequence AND depth logits
 *   out  [B,T,Hq,d]        out  attention output (input dtype)
 *   lse  [B,Hq,T] fp32     out  natural-log softmax denominator of the scaled
 *                               logits (needed by moda_bwd); may be NULL
 * Returns MODA_OK once the kernel is enqueued on `stream`.
 */
moda_status moda_fwd(const void* q, const void* k, const void* v,
                     const void* kd, const void* vd,
                     int B, int T, int Hq, int Hkv, int d, int Ld,
                     moda_dtype dtype, float scale,
                     void* out, float* lse, void* stream);

/* moda_fwd with an explicit kernel family (MODA_IMPL_SIMT forces the scalar
 * reference kernels; MODA_IMPL_TC requires a tensor-core-supported shape and
 * returns MODA_ERR_UNSUPPORTED otherwise). Same arguments and semantics. */
moda_status moda_fwd_ex(const void* q, const void* k, const void* v,
                        const void* kd, const void* vd,
                        int B, int T, int Hq, int Hkv, int d, int Ld,
                        moda_dtype dtype, float scale,
                        void* out, float* lse, void* stream, moda_impl impl);

/*
 * moda_fwd_sel — moda_fwd with a per-token selection of depth slots: the
 * bounded depth-KV slots ("sliding window" over layers or a dynamic choice of
 * layers) that "Mixture-of-Depths Attention" (gist.science German summary §5,
 * future directions) proposes for very deep models.
 *   depth_sel [B,T] uint64  in  device bit masks, 8-byte aligned: bit i of
 *                               depth_sel[b*T + t] set = token t's depth slot
 *                               i (kd[b,t,i], vd[b,t,i]) takes part in its
 *                               softmax; clear = that slot is absent for
 *                               every head of the token. Bits >= Ld are
 *                               ignored. NULL = every slot (= moda_fwd_ex).
 * A token whose mask is 0 attends to its causal sequence keys only (its own
 * key is always visible, so no row is empty). A non-NULL mask needs
 * Ld <= 64, else MODA_ERR_UNSUPPORTED. The depth keys of unselected slots are
 * still read (the kernels load whole tiles); only the result changes.
 * Other arguments, semantics and errors as moda_fwd_ex.
 */
moda_status moda_fwd_sel(const void* q, const void* k, const void* v,
                         const void* kd, const void* vd, const uint64_t* depth_sel,
                         int B, int T, int Hq, int Hkv, int d, int Ld,
                         moda_dtype dtype, float scale,
                         void* out, float* lse, void* stream, moda_impl impl);

/*
 * moda_bwd_workspace_bytes — bytes of fp32 scratch moda_bwd needs for this
 * shape: row statistics D [B,Hq,T] and, for bf16 (tensor-core path), fp32
 * accumulators of dk and dv [B,T,Hkv,d]. Returns 0 for an invalid shape.
 */
size_t moda_bwd_workspace_bytes(int B, int T, int Hq, int Hkv, int d, int Ld,
                                moda_dtype dtype);

/*
 * moda_bwd — gradients of moda_fwd for upstream gradient dout. The pages give
 * no backward pass; this is the derivative of the forward definition above:
 *   P = exp(s - lse), dP = [dout.v_j || dout.vd_i], D = sum P dP (over the
 *   row's sequence and depth keys), dS = P * (dP - D);
 *   dq = scale*(sum_j dS_j k_j + sum_i dS'_i kd_i),
 *   dk_j = scale*sum dS_j q, dv_j = sum P_j dout (over rows t >= j of the
 *   group's G heads), dkd / dvd likewise over the G heads of the same token.
 * D equals <dout, out> of the exact output. The library takes <dout, out>
 * of the output it is given only as a first estimate and corrects it from
 * its own recomputed P and dP, so the gradients do not inherit the rounding
 * of the stored (bf16) output, which wide depth keys would amplify.
 *   q,k,v,kd,vd,out   in   as in moda_fwd (out is moda_fwd's output)
 *   lse               in   moda_fwd's lse
 *   dout [B,T,Hq,d]   in   upstream gradient
 *   dq,dk,dv,dkd,dvd  out  gradients, input dtype, same layouts as the inputs
 *                          (dkd / dvd may be NULL iff Ld == 0)
 *   workspace         in   device scratch of >= moda_bwd_workspace_bytes(...)
 *                          bytes, 16-byte aligned; contents on entry ignored
 */
moda_status moda_bwd(const void* q, const void* k, const void* v,
                     const void* kd, const void* vd,
                     const void* out, const float* lse, const void* dout,
                     int B, int T, int Hq, int Hkv, int d, int Ld,
                     moda_dtype dtype, float scale,
                     void* dq, void* dk, void* dv, void* dkd, void* dvd,
                     void* workspace, size_t workspace_bytes, void* stream);

/* moda_bwd with an explicit kernel family; same arguments and semantics. */
moda_status moda_bwd_ex(const void* q, const void* k, const void* v,
                        const void* kd, const void* vd,
                        const void* out, const float* lse, const void* dout,
                        int B, int T, int Hq, int Hkv, int d, int Ld,
                        moda_dtype dtype, float scale,
                        void* dq, void* dk, void* dv, void* dkd, void* dvd,
                        void* workspace, size_t workspace_bytes, void* stream,
                        moda_impl impl);

/*
 * moda_bwd_sel — gradients of moda_fwd_sel: moda_bwd_ex with the same
 * depth_sel as the forward (out and lse must come from moda_fwd_sel with that
 * mask). Unselected depth slots get dkd = dvd = 0; the other gradients see
 * only the selected slots. depth_sel NULL = moda_bwd_ex.
 */
moda_status moda_bwd_sel(const void* q, const void* k, const void* v,
                         const void* kd, const void* vd, const uint64_t* depth_sel,
                         const void* out, const float* lse, const void* dout,
                         int B, int T, int Hq, int Hkv, int d, int Ld,
                         moda_dtype dtype, float scale,
                         void* dq, void* dk, void* dv, void* dkd, void* dvd,
                         void* workspace, size_t workspace_bytes, void* stream,
                         moda_impl impl);

/*
 * moda_bwd_noalloc — moda_bwd for callers that cannot allocate device memory.
 * The paper has no counterpart to this entry point: it serves how a program
 * embeds the library, not the MoDA method.
 *
 * Who needs it: a caller that owns no device allocator for this library, e.g.
 * a C / C++ host program that hands over only its input and output buffers,
 * or a runtime that reserves the whole device for its own memory pool, where
 * a library's cudaMalloc would fail once the pool has claimed the memory or
 * would bypass the runtime's accounting. Such a caller cannot supply the
 * workspace moda_bwd needs.
 *
 * What it does: the same gradients as moda_bwd (same arguments minus the
 * workspace, same layouts, same error codes), computed by the scalar (SIMT)
 * backward kernels, with the fp32 row statistics D[B, Hq, T] kept in a fixed
 * array of MODA_NOALLOC_SCRATCH_BYTES bytes compiled into the library. It
 * calls no cudaMalloc or cudaFree and no allocating routine.
 *   - Cost: every GPU that loads the library holds that array until exit.
 *   - Limit: B * Hq * T * 4 bytes must fit in the array; larger problems
 *     return MODA_ERR_WORKSPACE with nothing launched.
 *   - Set-up: the first call on each device resolves the array's device
 *     address (cudaGetSymbolAddress, with that device current). Make that
 *     first call before any stream capture on the device. The address is
 *     kept per CUDA context: after cudaDeviceReset (or a new primary
 *     context) the next call resolves it again, so make that call outside
 *     a capture too.
 *   - Sharing: every call on a device uses the same array, which keeps the
 *     previous call's contents (nothing needs clearing: the backward writes
 *     every entry before reading it). Calls whose kernels overlap on the GPU
 *     (different streams without ordering between them) race on the array;
 *     order them on one stream or with events.
 */
#define MODA_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
moda_status moda_bwd_noalloc(const void* q, const void* k, const void* v,
                             const void* kd, const void* vd,
                             const void* out, const float* lse, const void* dout,
                             int B, int T, int Hq, int Hkv, int d, int Ld,
                             moda_dtype dtype, float scale,
                             void* dq, void* dk, void* dv, void* dkd, void* dvd,
                             void* stream);

/*
 * moda_pack_depth — optional repack of the depth keys and values into the
 * flattened per-kv-head layout [2][B][Hkv][T*Ld][d] ("Mixture-of-Depths
 * Attention", gist.science German summary §2: depth KV flattened along one
 * T x L axis so that a flash-style kernel reads it blockwise; first half kd,
 * second half vd). moda_fwd reads the native layout directly, so this is
 * never needed for correctness; its cost is measured separately.
 *   kd, vd [B,T,Ld,Hkv,d]  in
 *   packed                 out  moda_pack_depth_bytes(...) bytes, 16-B aligned
 */
size_t moda_pack_depth_bytes(int B, int T, int Hkv, int d, int Ld, moda_dtype dtype);
moda_status moda_pack_depth(const void* kd, const void* vd,
                            int B, int T, int Hkv, int d, int Ld, moda_dtype dtype,
                            void* packed, void* stream);

/*
 * moda_depth_write — the method's write step ("Mixture-of-Depths Attention",
 * gist.science German summary §2, Write-Step): after a layer has run, its
 * key/value pairs (for an FFN layer, the pair its light projection produced)
 * are appended to the depth stream that later layers read. This copies
 *   kd[b, t, slot, h, :] = k[b, t, h, :]   and   vd[b, t, slot, h, :] = v[b, t, h, :]
 * for every b, t, h, in the native depth layout that moda_fwd reads, so no
 * repack is needed between layers; the other slots are left untouched.
 *   k, v   [B,T,Hkv,d]      in   the layer's keys / values (input dtype)
 *   kd, vd [B,T,Ld,Hkv,d]   in/out  the depth cache; slot `slot` is written
 *   slot                    in   0 <= slot < Ld, else MODA_ERR_INVALID_VALUE
 * All pointers 16-byte aligned (MODA_ERR_MISALIGNED); d * element size must
 * be a multiple of 16 bytes (MODA_ERR_UNSUPPORTED); k / v must not overlap
 * kd / vd. Bit-exact copy; enqueued on `stream`.
 */
moda_status moda_depth_write(const void* k, const void* v,
                             int B, int T, int Hkv, int d, int Ld, int slot,
                             moda_dtype dtype, void* kd, void* vd, void* stream);

/*
 * 8-bit depth KV. "动态混合深度注意力机制MoDA技术解析" (mhpn.cn) §4.2 suggests
 * storing the depth KV of deep models (beyond 32 layers) with 8-bit
 * quantisation where device memory is short; the page names no format. This
 * library's format: int8 codes in the native depth layout [B,T,Ld,Hkv,d] and
 * one fp32 scale per (b, t, slot, kv-head) row of d values [B,T,Ld,Hkv]:
 *     scale = amax / 127 (amax = max |x| over the row; 0 for a zero row),
 *     code  = round-half-even(x / scale) clamped to [-127, 127]  (0 if scale 0),
 * each step one IEEE fp32 operation. The depth value the forward attends to
 * is fp32(scale * code) rounded to the input dtype (round to nearest even
 * for bf16): the 8-bit cache decompresses into the type an unquantised depth
 * cache would hold. About half the bytes of the bf16 depth stream (d + 4
 * bytes per row instead of 2d).
 *
 * moda_depth_quantize_q8 — quantise a whole bf16 / fp32 depth cache.
 *   kd, vd [B,T,Ld,Hkv,d]             in   (input dtype)
 *   kd8, vd8 [B,T,Ld,Hkv,d] int8      out  16-byte aligned
 *   kd_scale, vd_scale [B,T,Ld,Hkv]   out  fp32, 4-byte aligned
 * moda_depth_write_q8 — the write step into an 8-bit cache: k, v [B,T,Hkv,d]
 *   quantised into slot `slot` (0 <= slot < Ld) of kd8 / vd8 and its scales;
 *   other slots untouched.
 * moda_fwd_q8 — moda_fwd_ex reading the 8-bit depth cache (codes and
 *   scales as above; all four may be NULL iff Ld == 0). The tensor-core path
 *   dequantises each depth tile in shared memory, the SIMT path per row in
 *   registers, to the same values. Forward only: there is no 8-bit backward.
 * Errors as moda_fwd_ex / moda_depth_write; MODA_ERR_MISALIGNED for a scale
 * pointer that is not 4-byte aligned.
 */
moda_status moda_depth_quantize_q8(const void* kd, const void* vd,
                                   int B, int T, int Hkv, int d, int Ld, moda_dtype dtype,
                                   int8_t* kd8, int8_t* vd8, float* kd_scale, float* vd_scale,
                                   void* stream);
moda_status moda_depth_write_q8(const void* k, const void* v,
                                int B, int T, int Hkv, int d, int Ld, int slot, moda_dtype dtype,
                                int8_t* kd8, int8_t* vd8, float* kd_scale, float* vd_scale,
                                void* stream);
moda_status moda_fwd_q8(const void* q, const void* k, const void* v,
                        const int8_t* kd8, const int8_t* vd8,
                        const float* kd_scale, const float* vd_scale,
                        int B, int T, int Hq, int Hkv, int d, int Ld,
                        moda_dtype dtype, float scale,
                        void* out, float* lse, void* stream, moda_impl impl);

/*
 * moda_depth_slot_layout — where a producer writes a layer's K / V so that
 * they land directly in slot `slot` of the native depth cache, with no copy
 * pass: the write step of "Mixture-of-Depths Attention" (gist.science German
 * summary §2, Write-Step) fused into whatever kernel produces the pair (the
 * layer's key / value projection, or an FFN layer's light projection).
 * Slot `slot` of kd [B,T,Ld,Hkv,d] is the strided tensor [B, T, Hkv, d] that
 * starts `*offset` elements after kd and has element strides
 *     strides[0..3] = {T*Ld*Hkv*d, Ld*Hkv*d, d, 1}     (b, t, h, feature)
 * so a GEMM producing the [B*T, Hkv*d] row block writes it with leading
 * dimension Ld*Hkv*d (vd likewise). moda_depth_write is the copy pass this
 * replaces. Returns MODA_ERR_INVALID_VALUE for a bad shape, slot or NULL
 * output pointer; touches no device.
 */
moda_status moda_depth_slot_layout(int B, int T, int Hkv, int d, int Ld, int slot,
                                   long long* offset, long long strides[4]);

/* moda_fwd reading depth keys/values from moda_pack_depth's layout. */
moda_status moda_fwd_packed(const void* q, const void* k, const void* v,
                            const void* packed_depth,
                            int B, int T, int Hq, int Hkv, int d, int Ld,
                            moda_dtype dtype, float scale,
                            void* out, float* lse, void* stream);

/*
 * moda_fwd_host — moda_fwd end to end from HOST buffers: enqueues on
 * `stream` the host-to-device copies of q, k, v, kd, vd into the caller's
 * device staging buffer, the forward on the staged inputs, and the
 * device-to-host copies of out and lse. No pages describe this; it is the
 * boundary a host program without device buffers of its own uses.
 * When the tensor-core forward serves the shape and T spans at least two of
 * its work units (2 * 128 / G tokens), the call pipelines up to 16 chunks of
 * query tokens: the copies of chunk j run on `stream` while the forward of
 * the chunks before it runs on a stream of the library's own and their
 * outputs are copied back on another (the causal mask makes a chunk's
 * queries need only the keys copied before it). `stream` waits for all of
 * it before any later work it holds; the result is the same bit for bit.
 *   q, k, v, kd, vd   in   HOST pointers, layouts as in moda_fwd (kd / vd NULL
 *                          iff Ld == 0)
 *   out, lse          out  HOST pointers (lse may be NULL)
 *   staging           in   DEVICE buffer of >= moda_fwd_host_staging_bytes(...)
 *                          bytes, 256-byte aligned; contents on entry ignored,
 *                          holds the staged tensors afterwards
 * Host buffers should be page-locked (cudaHostAlloc / cudaHostRegister) for
 * the copies to be asynchronous; with pageable memory the copies still work
 * but block the calling thread. Returns once everything is enqueued; out and
 * lse hold the results when the stream reaches the end of the call (e.g.
 * after moda_device_status(stream)). Errors: as moda_fwd, MODA_ERR_WORKSPACE
 * for a missing or short staging buffer, MODA_ERR_CUDA if a copy cannot be
 * enqueued. After an error that comes once copies or launches are enqueued,
 * `stream` is still ordered after all of them (else the call waits for them
 * before it returns), so the buffers may be released once `stream` is done;
 * out and lse are then undefined.
 */
size_t moda_fwd_host_staging_bytes(int B, int T, int Hq, int Hkv, int d, int Ld,
                                   moda_dtype dtype);
moda_status moda_fwd_host(const void* q, const void* k, const void* v,
                          const void* kd, const void* vd,
                          int B, int T, int Hq, int Hkv, int d, int Ld,
                          moda_dtype dtype, float scale,
                          void* out, float* lse,
                          void* staging, size_t staging_bytes, void* stream);

/*
 * moda_device_status — synchronises `stream`, then reads and clears the
 * device status word of the current device. Returns MODA_ERR_DEVICE_TIMEOUT if
 * a kernel's bounded wait expired since the last call, MODA_ERR_CUDA if the
 * synchronisation itself failed, else MODA_OK.
 */
moda_status moda_device_status(void* stream);

/*
 * moda_debug_set_wait_limit — test hook: caps every bounded on-chip wait of
 * later launches on the current device at `spins` polls (0 restores the
 * default, which is far above any legitimate wait). With a tiny cap a wait
 * that would succeed still expires, which exercises the timeout path without
 * faulting or hanging the GPU.
 */
moda_status moda_debug_set_wait_limit(uint32_t spins);

/*
 * moda_debug_exp2_poly — test hook: y[i] = 2^x[i] computed by the forward
 * kernel's FMA-pipe exponential (the share of the softmax exponentials that
 * does not go to the MUFU unit). x, y: device fp32 arrays of n elements.
 * Relative error <= 1e-4 for x in [-125, 16]; x < -125 gives ~2^-125.
 */
moda_status moda_debug_exp2_poly(const float* x, float* y, int n, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MODA_H_ */
