/*
 * nvnorm.h -- C ABI of the B200 (sm_100a) fused row-normalisation library, libnvnorm.so.
 *
 * Every op works row by row over the last axis of a contiguous row-major array
 * [rows, D] (rows = the product of the leading axes), with one element type for
 * all tensors of a call.  Arithmetic is float32 inside the kernels, with wider
 * arithmetic where a bfloat16 result would otherwise lose its last bit (layer_norm
 * statistics, the rope rotation); the results are rounded once, to nearest even.
 *
 * Ownership and memory
 *   - The caller owns every buffer.  The library allocates no memory, keeps no
 *     per-call state and has no handle.  All pointers are device (or managed)
 *     memory of the CURRENT device; each one is checked on the host against its
 *     allocation's extent before anything is launched.
 *   - Calls are asynchronous on `stream` (NULL = the legacy default stream); a
 *     return of NV_OK means the kernel was launched, not that it finished.
 *   - An output may be the very same buffer as an input (y == x, h == x, h == r):
 *     each row is read completely before it is written.  Any other overlap between
 *     an output and another buffer, and y == h, are rejected.
 *
 * Errors
 *   - Every argument is validated on the host before any launch; a failure
 *     returns NV_ERR_INVALID_ARG (or NV_ERR_UNSUPPORTED) and launches nothing.
 *   - rows == 0 is valid and launches nothing.
 *   - A launch failure reported by the CUDA runtime returns NV_ERR_CUDA.
 *   - nv_last_error() gives a message for the last non-OK status of the calling
 *     thread.  No C++ exception crosses this interface.
 *   - Invalid input values (Inf, NaN) are not errors: they propagate through the
 *     row that holds them, per IEEE arithmetic, and reach no other row.
 *
 * Scalars: eps, base and scale are float32 values, as the op definitions store them
 * (docs.rs nuvec-core 0.5.0, Enum FastOp: every field is f32::to_bits).
 */
#ifndef NVNORM_H
#define NVNORM_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NV_API __attribute__((visibility("default")))
#else
#define NV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream (the same handle as cudaStream_t / CUstream). */
typedef struct CUstream_st* nv_stream_t;

typedef enum {
    NV_F32 = 0,  /* IEEE binary32 */
    NV_BF16 = 1, /* bfloat16 */
    NV_F16 = 2   /* IEEE binary16: reserved, returns NV_ERR_UNSUPPORTED */
} nv_dtype;

typedef enum {
    NV_OK = 0,
    NV_ERR_INVALID_ARG = 1,
    NV_ERR_UNSUPPORTED = 2,
    NV_ERR_CUDA = 3
} nv_status;

/*
 * rms_norm -- docs.rs nuvec-core 0.5.0, Enum FastOp, variant RmsNorm:
 *   y = x / sqrt(mean(x^2) + eps) * w over the last axis; w is a length-D vector, or NULL for 1
 *   (nuvec-nn src/layers.rs, RmsNorm::forward; miniVLLM Layers page, LayerNorm with
 *   residual = None).
 * x [rows, D] in; w [D] in, or NULL for w = 1; y [rows, D] out (may be x).
 * rows >= 0, D >= 1, eps finite and >= 0.
 */
NV_API nv_status nv_rms_norm(const void* x, const void* w, void* y, int64_t rows, int64_t D, float eps,
                      nv_dtype dt, nv_stream_t stream);

/*
 * add_rms_norm -- docs.rs nuvec-core 0.5.0, Enum FastOp, variant AddRmsNorm:
 *   h = x + r and RmsNorm of h; miniVLLM Layers page, LayerNorm.forward with a
 *   residual (x_new = x + residual, normalise x_new, return (normalised, x_new)).
 * h is the float32 sum x + r rounded once to the I/O type, and y normalises exactly
 * that rounded h, so add_rms_norm(x, r) == rms_norm(h) bit for bit.
 * x, r [rows, D] in; w [D] in or NULL (w = 1); y [rows, D] out; h [rows, D] out.
 * h may be x or r; y may be x or r; y != h.
 */
NV_API nv_status nv_add_rms_norm(const void* x, const void* r, const void* w, void* y, void* h,
                          int64_t rows, int64_t D, float eps, nv_dtype dt, nv_stream_t stream);

/*
 * layer_norm -- docs.rs nuvec-core 0.5.0, Enum FastOp, variant LayerNorm:
 *   y = (x - mean) / sqrt(var + eps) * w + b over the last axis, w and b length-D
 *   vectors or NULL for 1 and 0 (nuvec-nn src/layers.rs, LayerNorm: affine / without_bias).
 * var is the population variance (sum of squared deviations / D).
 * x [rows, D] in; w [D] or NULL (w = 1); b [D] or NULL (b = 0); y [rows, D] out.
 */
NV_API nv_status nv_layer_norm(const void* x, const void* w, const void* b, void* y, int64_t rows,
                        int64_t D, float eps, nv_dtype dt, nv_stream_t stream);

/*
 * norm_rope -- docs.rs nuvec-core 0.5.0, Enum FastOp, variants NormRope and Rope
 * (non-cache form): every row (b, h, l) of x [B, H, L, D] is RMS-normalised with eps
 * and w, then its first dims features are rotated at position offset + l:
 *   theta_i = base^(-2 i / dims), phi_i = (offset + l) * scale * theta_i,
 *   (y_p, y_q) = (n_p cos phi_i - n_q sin phi_i, n_p sin phi_i + n_q cos phi_i)
 * for the pairs (p, q) = (i, i + dims/2) (traditional = 0: the two halves) or
 * (2i, 2i + 1) (traditional != 0: interleaved pairs).  Features j >= dims keep the
 * normalised value.  normalize == 0 is plain Rope: no normalisation, w and eps unused.
 * x [rows, D] in with rows = B*H*L (row k at l = k mod L); w [D] or NULL (w = 1);
 * y [rows, D] out (may be x).
 * L >= 1, rows % L == 0, dims even with 0 < dims <= D, base > 0 and finite, scale
 * finite, offset >= 0, eps finite and >= 0 (checked only when normalize != 0).
 */
NV_API nv_status nv_norm_rope(const void* x, const void* w, void* y, int64_t rows, int64_t L, int64_t D,
                       int32_t dims, int32_t traditional, float base, float scale, int64_t offset,
                       int32_t normalize, float eps, nv_dtype dt, nv_stream_t stream);

/*
 * rope -- the general form of norm_rope: docs.rs nuvec-core 0.5.0, Enum FastOp, variant
 * NormRope with its cache form (rotated rows land in the cache at their own positions) and
 * variant Rope with an explicit frequency vector and a direction.
 *   freqs    [dims/2] float32 device array of frequencies theta_i replacing
 *            base^(-2 i / dims) (base is then ignored), or NULL.
 *   forward  != 0: turn by +phi_i; 0: the inverse rotation (-phi_i), the gradient of Rope.
 *   y_len    0: y is [B, H, L, D] like x (may be x).  > 0: y is a cache [B, H, y_len, D]
 *            and row (b, h, l) of x is written to cache row (b, h, offset + l), at the
 *            same position offset + l it is rotated at; no other cache row is written.
 *            Requires y_len >= offset + L; y must not overlap x then.
 * Other arguments as nv_norm_rope; base is checked only when freqs is NULL.
 */
NV_API nv_status nv_rope(const void* x, const void* w, const float* freqs, void* y, int64_t rows,
                         int64_t L, int64_t y_len, int64_t D, int32_t dims, int32_t traditional,
                         float base, float scale, int64_t offset, int32_t forward,
                         int32_t normalize, float eps, nv_dtype dt, nv_stream_t stream);

/*
 * rms_norm_vjp -- docs.rs nuvec-core 0.5.0, Enum FastOp, variant RmsNormVjp: the
 * gradients of rms_norm for x and w.  With r = 1/sqrt(mean(x^2) + eps):
 *   dx_j = r w_j g_j - x_j r^3 (sum_k g_k w_k x_k) / D,   dw_j = sum over rows of g_j x_j r.
 * x, g [rows, D] in (g = the gradient of y); w [D] in or NULL (w = 1); dx [rows, D] out
 * (may be x or g); dw [D] out, given exactly when w is (w = 1 has no gradient).
 * workspace: device memory of at least nv_norm_vjp_workspace_size(0, rows, D) bytes when
 * dw is requested (per-CTA partial sums of the columns; contents are overwritten), else
 * may be NULL.  dw is deterministic: the partials are added in a fixed order in double.
 * rows == 0 with dw requested writes dw = 0.  Any D >= 1 and any element alignment: rows
 * of whole 16-byte vectors with D <= 16384 (bf16) / 8192 (f32) and 16-byte aligned x, g, dx
 * and w take the register kernels; other rows a generic kernel (scalar accesses, row
 * statistics in double; slower).
 */
NV_API nv_status nv_rms_norm_vjp(const void* x, const void* w, const void* g, void* dx, void* dw,
                                 void* workspace, size_t workspace_bytes, int64_t rows, int64_t D,
                                 float eps, nv_dtype dt, nv_stream_t stream);

/*
 * layer_norm_vjp -- docs.rs nuvec-core 0.5.0, Enum FastOp, variant LayerNormVjp: the
 * gradients of layer_norm for x, w and b (b itself does not enter them).  With
 * r = 1/sqrt(var + eps), xh = (x - mean) r, a = w g:
 *   dx_j = r (a_j - mean(a) - xh_j mean(a xh)),  dw_j = sum_rows g_j xh_j,  db_j = sum_rows g_j.
 * dw given exactly when w is; db [D] out or NULL.  workspace: at least
 * nv_norm_vjp_workspace_size(2, rows, D) bytes when dw or db is requested.  Otherwise as
 * nv_rms_norm_vjp.
 */
NV_API nv_status nv_layer_norm_vjp(const void* x, const void* w, const void* g, void* dx,
                                   void* dw, void* db, void* workspace, size_t workspace_bytes,
                                   int64_t rows, int64_t D, float eps, nv_dtype dt,
                                   nv_stream_t stream);

/* Workspace bytes for the vjp column sums (op 0 rms_norm_vjp, 2 layer_norm_vjp; 0 for
 * invalid arguments). */
NV_API size_t nv_norm_vjp_workspace_size(int32_t op, int64_t rows, int64_t D);

/*
 * rope_llama3_freqs -- the Llama 3 long-context frequency scaling ("NTK-by-parts") for
 * nv_rope's `freqs`: miniVLLM Layers page, section RotaryEmbedding, parameters
 * llama3_rope_factor (scales the low-frequency components), llama3_rope_low_freq_factor and
 * llama3_rope_high_freq_factor (wavelength thresholds original_max_position / factor) and
 * llama3_rope_original_max_position_embeddings; docs.rs nuvec-core 0.5.0, Enum FastOp,
 * variant Rope (frequency scaling by Llama3RoPE).  The pages print no formula; read as:
 * with theta_i = base^(-2i/dims) and wavelength 2 pi / theta_i, wavelengths below
 * original_max_position / high_freq_factor keep theta_i, those above
 * original_max_position / low_freq_factor get theta_i / factor, and between them
 * (1 - s) theta_i / factor + s theta_i with s = (original_max_position / wavelength -
 * low_freq_factor) / (high_freq_factor - low_freq_factor).  Computed in double on the host,
 * rounded once: freqs [dims / 2] is HOST memory (copy it to the device for nv_rope).
 * Needs dims even >= 2, base > 0, factor >= 1, 0 < low_freq_factor < high_freq_factor,
 * original_max_position > 0 (else NV_ERR_INVALID_ARG).  Needs no GPU.
 */
NV_API nv_status nv_rope_llama3_freqs(int32_t dims, float base, float factor,
                                      float low_freq_factor, float high_freq_factor,
                                      int64_t original_max_position, float* freqs);

/*
 * rope_yarn_freqs -- YaRN frequency scaling for nv_rope's `freqs`: docs.rs nuvec-core 0.5.0,
 * Enum FastOp, variant Rope names it (frequency scaling by YarnRoPE) without parameters or
 * formula; read as the published method (Peng, Quesnelle, Fan and Shippole, "YaRN:
 * Efficient Context Window Extension of Large Language Models", 2023).  With
 * theta_i = base^(-2i/dims), pair i turns r_i = original_max_position * theta_i / (2 pi)
 * times over the original context; pairs with r_i > beta keep theta_i, pairs with
 * r_i < alpha get theta_i / factor, and between them theta_i / factor is blended linearly
 * toward theta_i by (r_i - alpha) / (beta - alpha) ("NTK-by-parts").  YaRN also scales the
 * rotated q and k each by the temperature factor mscale = 0.1 ln(factor) + 1; this library
 * does not apply it: multiply the attention logits by mscale^2 (or q and k by mscale).
 * The paper's values for LLaMA are alpha = 1, beta = 32.  Computed in double on the host,
 * rounded once: freqs [dims / 2] and mscale are HOST memory (copy freqs to the device for
 * nv_rope); mscale may be NULL.  Needs dims even >= 2, base > 0, factor >= 1,
 * 0 < alpha < beta, original_max_position > 0 (else NV_ERR_INVALID_ARG).  Needs no GPU.
 */
NV_API nv_status nv_rope_yarn_freqs(int32_t dims, float base, float factor,
                                    int64_t original_max_position, float alpha, float beta,
                                    float* freqs, float* mscale);

/*
 * rope_suscaled_freqs -- SuScaled (LongRoPE) frequency scaling for nv_rope's `freqs`:
 * docs.rs nuvec-core 0.5.0, Enum FastOp, variant Rope names it (frequency scaling by
 * SuScaledRoPE) without parameters or formula; read as the published method (Ding et al.,
 * "LongRoPE: Extending LLM Context Window Beyond 2 Million Tokens", 2024) in the form of the
 * Phi-3 models (Abdin et al., "Phi-3 Technical Report", 2024).  Every pair i has its own
 * rescale factor lambda_i and turns at theta_i / lambda_i, theta_i = base^(-2i/dims); the
 * factors are long_factors when seq_len > original_max_position, else short_factors.
 * Extending the original context L to max_position L' also scales the rotated q and k by
 * the attention factor mscale = sqrt(1 + ln(L'/L) / ln L) when L' > L (1 otherwise); this
 * library does not apply it (multiply q and k, or the logits by its square).
 * short_factors, long_factors [dims / 2], freqs [dims / 2] and mscale are HOST memory
 * (copy freqs to the device for nv_rope); mscale may be NULL.  Computed in double on the
 * host, rounded once.  Needs dims even >= 2, base > 0, the chosen factors finite and > 0,
 * original_max_position >= 2, max_position >= 1, seq_len >= 0 (else NV_ERR_INVALID_ARG).
 * Needs no GPU.
 */
NV_API nv_status nv_rope_suscaled_freqs(int32_t dims, float base, const float* short_factors,
                                        const float* long_factors, int64_t seq_len,
                                        int64_t max_position, int64_t original_max_position,
                                        float* freqs, float* mscale);

/*
 * allreduce_add_rms_norm -- the step a tensor-parallel decoder takes after a row-parallel
 * layer: miniVLLM Layers page, section Linear layers, RowParallelLinear (the forward pass
 * sums the ranks' partial outputs with an all_reduce), then the fused residual add +
 * RMSNorm (same page, section LayerNorm; docs.rs nuvec-core 0.5.0, Enum FastOp, variant
 * AddRmsNorm).  This call is the reduction half of a one-shot all-reduce fused with the
 * norm: given every rank's partial output it computes
 *   x = sum of parts[0..nparts) in that order, in double, rounded once to dt;
 *   h = x + r in float32 rounded to dt;  y = h / sqrt(mean(h^2) + eps) * w.
 * Every rank that calls it with the same parts gets bit-identical x, h and y.
 * parts: host array of nparts (1..8) device pointers, each [rows, D] in: this GPU's memory
 * (for example the slots of an all-gather) or another GPU's buffer mapped into this
 * process (peer access / IPC; the call reads it directly).  r [rows, D] in (the residual);
 * w [D] or NULL; y [rows, D] out; h [rows, D] out (may be r); x_out [rows, D] out or NULL
 * (may be one of the parts).  r, w, y, h and x_out must be memory of the current device.
 * The caller orders the producers of remote parts before this call (e.g. a barrier or a
 * collective on `stream`).  Errors: NV_ERR_INVALID_ARG for bad pointers, sizes, overlaps or
 * nparts outside 1..8.
 */
NV_API nv_status nv_allreduce_add_rms_norm(const void* const* parts, int32_t nparts,
                                           const void* r, const void* w, void* y, void* h,
                                           void* x_out, int64_t rows, int64_t D, float eps,
                                           nv_dtype dt, nv_stream_t stream);

/*
 * allreduce_add_rms_norm_peers -- the one-shot form of nv_allreduce_add_rms_norm for ranks
 * that read each other's partials directly (same page and sections).  Every rank keeps its
 * partial output in its own device buffer, which the other ranks have mapped into their
 * processes (nv_ipc_export / nv_ipc_import), and a flag array of one int64 per rank in its
 * own device memory, also mapped by the others.  Per step `epoch` (1, 2, 3, ... on every
 * rank in lockstep) each rank, after producing its partial on `stream`, calls
 * nv_tp_publish, which stores `epoch` into its slot of every rank's flag array; then this
 * call waits on the device until every slot of this rank's `flags` [nparts] has reached
 * `epoch` and computes exactly what nv_allreduce_add_rms_norm computes, reading the parts
 * (this rank's own buffer and the mapped peers', in rank order) with plain loads.  The wait
 * is bounded (about a second per CTA): if a peer never publishes, each CTA that gave up
 * counts a fault (nv_fault_count) and leaves its rows unwritten; no error is returned by the
 * launch itself.  A rank must not overwrite the partial of step e before every rank's call
 * of step e has read it: write step e + 1 into a second buffer (double buffering) on the
 * same stream, after this call -- a peer then publishes e + 1 only after its own step-e call
 * has finished, and this rank's step e + 1 call waits for that before step e + 2 reuses the
 * first buffer.  flags: 8-byte aligned device memory of the current device, zero before the
 * first step.  Errors: as nv_allreduce_add_rms_norm, plus NV_ERR_INVALID_ARG for a NULL or
 * misaligned flags array or epoch < 1.
 */
NV_API nv_status nv_allreduce_add_rms_norm_peers(const void* const* parts, int32_t nparts,
                                                 const void* r, const void* w, void* y, void* h,
                                                 void* x_out, int64_t rows, int64_t D, float eps,
                                                 nv_dtype dt, const int64_t* flags, int64_t epoch,
                                                 nv_stream_t stream);

/*
 * tp_publish -- the publishing half of nv_allreduce_add_rms_norm_peers: after everything
 * queued on `stream` before it (this rank's partial of step `epoch`) has completed, a
 * system-scope fence and then one release store of `epoch` into slot `rank` of each of the
 * `world` flag arrays (flags[p]: rank p's array of `world` int64, this rank's own or a mapped
 * peer's).  world 1..8, 0 <= rank < world, epoch >= 1, each flags[p] 8-byte aligned device
 * memory (else NV_ERR_INVALID_ARG).
 */
NV_API nv_status nv_tp_publish(int64_t* const* flags, int32_t world, int32_t rank, int64_t epoch,
                               nv_stream_t stream);

/* Bytes of a device-memory handle for another process (cudaIpcMemHandle_t). */
#define NV_IPC_HANDLE_BYTES 64

/*
 * ipc_export / ipc_import / ipc_close -- sharing device buffers between the processes of
 * one node (CUDA IPC), for nv_allreduce_add_rms_norm_peers.  nv_ipc_export writes the
 * handle (NV_IPC_HANDLE_BYTES bytes, host memory) of the allocation holding `ptr` and the
 * offset of `ptr` inside it; another process passes both to nv_ipc_import, which maps the
 * allocation (with peer access enabled on demand) and returns the matching pointer there,
 * and later to nv_ipc_close with that pointer.  The handle is plain bytes: send it over
 * any channel (for example a process-group all-gather of objects).  Errors: NV_ERR_INVALID_ARG
 * for NULL arguments or a pointer outside any allocation, NV_ERR_CUDA when the runtime
 * refuses (for example importing a handle in the process that exported it).
 */
NV_API nv_status nv_ipc_export(const void* ptr, void* handle, uint64_t* offset);
NV_API nv_status nv_ipc_import(const void* handle, uint64_t offset, void** ptr);
NV_API nv_status nv_ipc_close(void* ptr, uint64_t offset);

/*
 * add_rms_norm_host -- add_rms_norm (as nv_add_rms_norm) on rows that live in host
 * memory: x and r are copied in, the op runs, y and h are copied back, pipelined over
 * chunks of chunk_rows rows (0 = about eight chunks, at most 64) through three internal
 * streams -- copies in, compute, copies out, linked per chunk by events -- so that copies
 * in and out and the compute of different chunks overlap.
 * x_host, r_host [rows, D] in, y_host, h_host [rows, D] out: page-locked host memory
 * (cudaHostAlloc / cudaHostRegister); y_host may be x_host and h_host may be r_host, other
 * host buffers may not overlap.  x_dev, r_dev, y_dev, h_dev [rows, D]: device buffers of
 * the current device owned by the caller, used as the staging area (on return their
 * contents are the inputs and outputs of the op; y_dev may be x_dev, h_dev may be r_dev).
 * w [D] device or NULL.  Asynchronous with respect to the host like the other calls: the
 * work starts after what is already queued on `stream`, and `stream` waits for all of it.
 * Calls from several host threads are serialised while they enqueue.  Errors as
 * nv_add_rms_norm, plus NV_ERR_INVALID_ARG for host buffers that are not page-locked.
 */
NV_API nv_status nv_add_rms_norm_host(const void* x_host, const void* r_host, const void* w,
                                      void* y_host, void* h_host, void* x_dev, void* r_dev,
                                      void* y_dev, void* h_dev, int64_t rows, int64_t D,
                                      float eps, nv_dtype dt, int64_t chunk_rows,
                                      nv_stream_t stream);

/*
 * rms_norm_vjp_static -- nv_rms_norm_vjp for callers that cannot allocate device memory.
 * The op definitions this library follows have no counterpart of this entry point: it
 * exists for callers that are handed their input and output buffers and may not allocate
 * more -- a plugin inside an inference engine or graph runtime that owns all memory, code
 * under a fixed memory budget, or a hot loop where cudaMalloc would synchronise the
 * device.  The caller passes x, w, g, dx and dw exactly as for nv_rms_norm_vjp, but no
 * workspace: the per-CTA partial sums of dw go to a fixed 4 MiB array in device memory
 * that the library declares (every GPU that loads the library holds it until the process
 * exits).  Nothing is allocated, and nothing needs clearing: each call writes every
 * partial row it later reads.
 *   - Limits: D <= 16384, D a multiple of 16 bytes of elements (8 bf16, 4 float32),
 *     float32 D <= 8192, 16-byte aligned x, g, dx and w (the register kernels only);
 *     other shapes return NV_ERR_UNSUPPORTED.  The number of partial rows is
 *     min(rows, SMs x resident CTAs per SM, max(512, 2^21 / D), 2^20 / D) -- at most
 *     2^20 / D, which is 64 at D = 16384 -- so dw can differ from nv_rms_norm_vjp's in the
 *     last bits (another summation grouping); dx is the same.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call before any
 *     stream capture.  The address is kept per device and CUDA context: after a device
 *     reset (a new context) the next call looks it up again.
 *   - All calls share the one array: two calls whose kernels overlap on the GPU (on
 *     different streams without ordering) race and may corrupt each other's dw.
 */
NV_API nv_status nv_rms_norm_vjp_static(const void* x, const void* w, const void* g, void* dx,
                                        void* dw, int64_t rows, int64_t D, float eps,
                                        nv_dtype dt, nv_stream_t stream);

/* Name of a status code (static storage). */
NV_API const char* nv_status_string(nv_status status);

/* Message for the calling thread's last non-OK status ("" if none yet). */
NV_API const char* nv_last_error(void);

/* Library version, major * 10000 + minor * 100 + patch. */
NV_API int32_t nv_version(void);

/*
 * Pointer checks -- by default every call asks the driver, for each pointer, whether it
 * is device memory of the current device and how far its allocation extends (one query per
 * pointer, a few tenths of a microsecond each; together most of the host time of a call on
 * a decode-sized batch).  A caller that guarantees its pointers -- buffers it allocated
 * itself, sized for the call, on the current device -- may turn these queries off for the
 * whole process with enabled = 0, and back on with 1.  Everything else is still checked:
 * sizes, NULL pointers, and the overlap of outputs with other buffers.  With the queries
 * off, a wrong pointer is no longer caught on the host: the kernel then reads or writes
 * whatever memory it is given.  previous: out, the former setting (1 on, 0 off), or NULL.
 * Always NV_OK.
 */
NV_API nv_status nv_set_pointer_checks(int32_t enabled, int32_t* previous);

/*
 * Device-side bounded waits that ran out, on the current device, since the library
 * was loaded (or last reset).  Only the staged kernels wait on the copy engine (and
 * nv_selftest_bounded_wait, on purpose, on a barrier nothing completes); each wait gives
 * up after about one second, counts a fault here, lets its copies in flight land and
 * leaves the rest of its rows unwritten.  Synchronises the device.
 * count: out, non-NULL.  reset != 0 sets the counter back to zero after reading it.
 */
NV_API nv_status nv_fault_count(uint32_t* count, int32_t reset);

/*
 * Check of the failure path of those bounded waits, for tests: launches `ctas` CTAs of
 * 32 threads on `stream`, each waiting on an mbarrier that nothing ever completes (no
 * copy is issued).  Every wait gives up after about one second and each CTA counts one
 * fault, so nv_fault_count then reports `ctas` more; nothing else is touched and the
 * context stays usable.  Takes about a second of GPU time.
 * ctas: 1..64.  Errors: NV_ERR_INVALID_ARG outside that range (nothing launched);
 * NV_ERR_CUDA on a launch error.
 */
NV_API nv_status nv_selftest_bounded_wait(int32_t ctas, nv_stream_t stream);

/*
 * Kernel-variant control, for tests and benchmarks.  The plain entry points above
 * pick a variant from (op, dtype, D, rows, alignment); the *_ex forms take a plan
 * that forces one.  A plan that the shape cannot use returns NV_ERR_UNSUPPORTED.
 *   path            NV_PATH_AUTO, or one of the kernel families below
 *   vec_per_thread  16-byte vectors per thread and row (register paths; 0 = auto; for
 *                   norm_rope 1 = one vector per lane, 2 = two vectors per lane (both
 *                   halves of a rotation, or two vectors of interleaved pairs), which
 *                   needs dims == D, or with dims < D rotated features that fill an even
 *                   number of whole 16-byte vectors and 4, 8 or 16 lanes per row)
 *   threads_per_row threads that share one row (multiple of 32, <= 1024; 0 = auto)
 *   rows_per_cta    rows one CTA works on at a time (0 = auto)
 *   ctas_per_sm     0: one CTA per row group (rms_norm register path, generic paths),
 *                   as many CTAs per SM as fit (layer_norm register path) or one CTA
 *                   per SM (staged path); > 0: a persistent grid of that many CTAs per
 *                   SM walking the rows
 *   launch          NV_LAUNCH_DEFAULT: programmatic dependent launch -- the kernel may
 *                   be scheduled while the preceding kernel of the stream finishes, and
 *                   it waits for that kernel (griddepcontrol.wait) before reading or
 *                   writing any global memory, so results are the same as with a plain
 *                   launch; NV_LAUNCH_PLAIN: ordinary stream-ordered launch.
 *   stages          NV_PATH_RING: shared-memory row buffers per CTA (0 = as many as fit,
 *                   at most 32; a multiple of rows_per_cta, at least 2 x rows_per_cta).
 *                   NV_PATH_SLOTS: 1 or 0 = each row slot asks L2 for its next row once
 *                   its current row has landed (one bulk prefetch a row); -1 = no
 *                   prefetch.  norm_rope register path
 *                   with two vectors per lane of 4, 8 or 16 lanes: 2..6 = that many rounds
 *                   of rows in flight per lane group, staged by per-thread asynchronous
 *                   copies into shared memory; -1 = rows in flight in registers; 0 =
 *                   automatic: with dims == D 2 rounds for bfloat16, registers for
 *                   float32; with dims < D 3 rounds for bfloat16, 4 for float32.
 *                   Other paths: must be 0.
 * For NV_PATH_RING, threads_per_row is the size of a row group (32 x warps, <= 256),
 * rows_per_cta the row groups of a CTA (rows reduced at once), ctas_per_sm the CTAs per
 * SM (0 = 1), vec_per_thread must be 0.
 */
typedef enum {
    NV_PATH_AUTO = 0,
    NV_PATH_ROWS = 1,    /* row held in registers, 16-byte vector loads */
    NV_PATH_GENERIC = 2, /* any D and alignment: scalar loop, two passes over the row */
    NV_PATH_STAGED = 3,  /* persistent, rows staged in shared memory by bulk async copies;
                            rms_norm, add_rms_norm and layer_norm.  rows_per_cta = rows in
                            flight per CTA (shared-memory stages), ctas_per_sm = CTAs per SM */
    NV_PATH_RING = 4,    /* layer_norm: persistent CTAs of several row groups (a few warps
                            each, reducing one row at a time) fed by a ring of shared-memory
                            row buffers that bulk async copies refill as rows finish */
    NV_PATH_SLOTS = 5    /* layer_norm, bfloat16: rows in registers, rows_per_cta of them per
                            persistent CTA sharing a float32 table of w and b in shared
                            memory; x consumed packed (bfloat16 -> double conversions and
                            mixed-precision fma, no unpacking) */
} nv_path;

typedef enum { NV_LAUNCH_DEFAULT = 0, NV_LAUNCH_PLAIN = 1 } nv_launch;

typedef struct {
    int32_t path;
    int32_t vec_per_thread;
    int32_t threads_per_row;
    int32_t rows_per_cta;
    int32_t ctas_per_sm;
    int32_t launch;
    int32_t stages;
} nv_plan;

NV_API nv_status nv_rms_norm_ex(const void* x, const void* w, void* y, int64_t rows, int64_t D,
                         float eps, nv_dtype dt, nv_stream_t stream, const nv_plan* plan);
NV_API nv_status nv_add_rms_norm_ex(const void* x, const void* r, const void* w, void* y, void* h,
                             int64_t rows, int64_t D, float eps, nv_dtype dt, nv_stream_t stream,
                             const nv_plan* plan);
NV_API nv_status nv_layer_norm_ex(const void* x, const void* w, const void* b, void* y, int64_t rows,
                           int64_t D, float eps, nv_dtype dt, nv_stream_t stream,
                           const nv_plan* plan);
NV_API nv_status nv_rope_ex(const void* x, const void* w, const float* freqs, void* y,
                            int64_t rows, int64_t L, int64_t y_len, int64_t D, int32_t dims,
                            int32_t traditional, float base, float scale, int64_t offset,
                            int32_t forward, int32_t normalize, float eps, nv_dtype dt,
                            nv_stream_t stream, const nv_plan* plan);
NV_API nv_status nv_norm_rope_ex(const void* x, const void* w, void* y, int64_t rows, int64_t L,
                          int64_t D, int32_t dims, int32_t traditional, float base, float scale,
                          int64_t offset, int32_t normalize, float eps, nv_dtype dt,
                          nv_stream_t stream, const nv_plan* plan);

/*
 * The plan that the plain entry point would use for these arguments (for reports).
 * op: 0 rms_norm, 1 add_rms_norm, 2 layer_norm, 3 norm_rope.  Returns NV_OK and
 * fills *plan, or an error status as the op itself would for invalid sizes.  For
 * norm_rope, D is the row length and dims/traditional are not considered; pointer
 * alignment is assumed to be 16 bytes.
 */
NV_API nv_status nv_describe_plan(int32_t op, int64_t rows, int64_t D, nv_dtype dt, nv_plan* plan);

#ifdef __cplusplus
}
#endif

#endif /* NVNORM_H */
