/*
 * dora.h -- C ABI of the B200 (sm_100a) DoRA adapter-layer library.
 *
 * One DoRA-adapted linear layer: frozen weight W0 [d_out x d_in], LoRA factors
 * A [r x d_in] and B [d_out x r], scale s and magnitude m [d_out]:
 *
 *     V' = W0 + s * B A,   C_i = ||V'_i|| (one norm per output row),
 *     y  = x (diag(m / C) V')^T
 *
 * Calls: dora_norm, dora_forward, dora_backward (the layer step);
 * dora_backward_full (without the norm's detach), dora_merge (deployment
 * weight), dora_vera_compose / dora_vera_grad (DVoRA); workspace sizing,
 * device status, a failure-detection self-test and kernel timing.
 *
 * Sources: "DoRA 阅读笔记" (zhongzhuzhou.org reading notes on DoRA, arXiv
 * 2402.09353) eq. (1), eq. (6), Algorithm 1, eq. (7), eq. (8), sections 3.4
 * and 3.5, appendix A;
 * "Scaling DoRA" (gptget.net/papers/2603.22276) English abstract: the row-wise
 * norm of W + sBA, its factored form (base + cross + Gram terms, no dense B A
 * product), and the fused single-pass composition in a form that is stable
 * when m / C is near 1.
 *
 * Conventions for every call
 *   - Device pointers on the current CUDA device; the caller owns every buffer.
 *     The library allocates nothing: scratch comes from the caller's workspace
 *     `ws` of at least dora_workspace_size() bytes (device memory, any content).
 *   - Row-major, contiguous. Tensors take desc->dtype (bf16 or fp32); m, norm,
 *     g, gm1 and dm are always fp32.
 *   - bf16: d_out, d_in and r must be multiples of 8, 8 <= r <= 512, and every
 *     pointer 16-byte aligned (TMA). fp32: any positive sizes, 4-byte aligned.
 *     T (tokens) may be any value >= 0; with T = 0 the per-token tensors (x, y,
 *     su_save, pre_save, dy, dx) may be NULL and the gradients are zero.
 *   - Each call only enqueues work on `stream` and returns; it does not
 *     synchronise. Outputs are overwritten, never accumulated into.
 *   - Non-finite inputs propagate as IEEE values; a zero norm gives inf/NaN.
 *   - A bad argument returns DORA_EINVAL before anything is launched; a launch
 *     failure returns DORA_ECUDA. dora_last_error() gives the message.
 */
#ifndef DORA_H_
#define DORA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DORA_API __attribute__((visibility("default")))
#else
#define DORA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* dora_stream_t;

typedef enum {
  DORA_OK = 0,
  DORA_EINVAL = 1,        /* null pointer, bad size, misalignment, bad dtype      */
  DORA_EUNSUPPORTED = 2,  /* valid request the library does not serve (r > 512, no sm_100 device) */
  DORA_EWORKSPACE = 3,    /* ws_bytes below dora_workspace_size()                 */
  DORA_ECUDA = 4,         /* a CUDA call or kernel launch failed                  */
  DORA_ETIMEOUT = 5       /* a kernel's bounded wait ran out (see dora_device_status) */
} dora_status_t;

typedef enum { DORA_BF16 = 0, DORA_FP32 = 1 } dora_dtype_t;

typedef enum {
  DORA_OP_NORM = 0,
  DORA_OP_FORWARD = 1,
  DORA_OP_BACKWARD = 2,
  DORA_OP_MERGE = 3,
  DORA_OP_BACKWARD_FULL = 4,
  DORA_OP_VERA_GRAD = 5
} dora_op_t;

typedef struct {
  int64_t d_out;      /* output features (rows of W0, B, entries of m)   */
  int64_t d_in;       /* input features (columns of W0 and A)            */
  int64_t r;          /* LoRA rank                                       */
  dora_dtype_t dtype; /* storage and operand type of the tensors         */
  float s;            /* LoRA scale (alpha / r)                          */
} dora_desc_t;

/* Bytes of workspace the call `op` needs for this layer and token count
 * (T is ignored for DORA_OP_NORM). Returns 0 for an invalid descriptor. */
DORA_API size_t dora_workspace_size(const dora_desc_t* desc, int64_t T, int op);

/*
 * dora_norm -- per-row norm of the adapted weight and the DoRA scale.
 *
 *   norm_out[i] = C_i = sqrt(max(0, ||W0_i||^2 + 2 s B_i (W0 A^T)_i + s^2 B_i (A A^T) B_i^T))
 *   g_out[i]    = m_i / C_i
 *   gm1_out[i]  = (m_i - C_i) / C_i        (g - 1 without cancellation)
 *
 * Scaling DoRA abstract (factored norm: base, cross and Gram terms; the dense
 * B A product is never formed); DoRA notes eq. (6) and Algorithm 1 step 9.
 * In:  W0 [d_out x d_in], A [r x d_in], B [d_out x r] (dtype); m [d_out] fp32.
 * Out: norm_out, g_out, gm1_out [d_out] fp32 (none may be NULL).
 */
DORA_API dora_status_t dora_norm(const dora_desc_t* desc, const void* W0, const void* A, const void* B,
                        const float* m, float* norm_out, float* g_out, float* gm1_out, void* ws,
                        size_t ws_bytes, dora_stream_t stream);

/*
 * dora_norm_noalloc -- dora_norm without a workspace argument; it allocates nothing.
 *
 * The pages describe no such call; it exists for callers that cannot allocate
 * device memory or hand over a workspace: applications whose memory manager
 * already owns the device memory they may use, loops that must not trigger
 * cudaMalloc's implicit synchronisation, and thin bindings that hold only the
 * layer's tensors. Same inputs, outputs and results as dora_norm.
 * Scratch: one 16 MiB (16,777,216-byte) device array inside the library, held
 * by every GPU that loads it until the process exits. A layer whose norm needs
 * more scratch than that (dora_workspace_size(desc, 0, DORA_OP_NORM) > 16 MiB)
 * is rejected with DORA_EUNSUPPORTED before anything is launched.
 * The first call on a device looks up the array's device address with that
 * device current and caches it; make that first call before any stream
 * capture. The cached address belongs to the device's current context: after
 * cudaDeviceReset() the process must load the library again before calling
 * this function on that device. All calls on a device share the array and
 * leave their contents in it (each call writes every scratch byte before
 * reading it): calls whose kernels may overlap on the GPU race and must be
 * ordered by the caller.
 */
DORA_API dora_status_t dora_norm_noalloc(const dora_desc_t* desc, const void* W0, const void* A, const void* B,
                                         const float* m, float* norm_out, float* g_out, float* gm1_out,
                                         dora_stream_t stream);

/*
 * dora_forward -- y = x (diag(g) V')^T for T tokens, composed in one pass.
 *
 *   su  = s * x A^T                                   [T x r]
 *   pre = x W0^T + su B^T  = x V'^T   (fp32, never rounded before use)
 *   y   = pre + gm1 (.) pre           (= g (.) pre; gm1 broadcast over tokens)
 *
 * DoRA notes eq. (6), Algorithm 1 steps 7-11; Scaling DoRA abstract (fused
 * single-pass composition, stable near g = 1). gm1 comes from dora_norm.
 * In:  x [T x d_in], W0, A, B (dtype); gm1 [d_out] fp32.
 * Out: y [T x d_out] (dtype).
 *      su_save [T x r] (dtype) receives s * x A^T; NULL keeps it in the workspace.
 *      pre_save [T x d_out] (dtype) receives pre, rounded once; NULL skips it.
 *      dora_backward needs both su_save and pre_save.
 */
DORA_API dora_status_t dora_forward(const dora_desc_t* desc, int64_t T, const void* x, const void* W0, const void* A,
                           const void* B, const float* gm1, void* y, void* su_save, void* pre_save, void* ws,
                           size_t ws_bytes, dora_stream_t stream);

/*
 * dora_backward -- gradients of the layer with the norm treated as a constant.
 *
 *   dz = g (.) dy                         (DoRA notes eq. (7): grad V' = (m / C) grad W')
 *   dm_i = sum_t dy[t,i] pre[t,i] / C_i    (eq. (8): grad W'_i . V'_i / ||V'_i||)
 *   dB = dz^T su,  du = s dz B,  dA = du^T x,  dx = dz W0 + du A
 *
 * The detach of DoRA notes section 3.4 and Algorithm 1 step 9: C carries no
 * gradient. W0 is frozen and gets none.
 * In:  dy [T x d_out], x [T x d_in], W0, A, B (dtype); norm = C and g [d_out]
 *      fp32 from dora_norm; su_save and pre_save from dora_forward (required).
 * Out: dm [d_out] fp32; dA [r x d_in], dB [d_out x r] (dtype);
 *      dx [T x d_in] (dtype) or NULL to skip the input gradient.
 * Streams: for small token batches the call may run dB and dA (or dx) on a
 * second stream owned by the library (one per host thread and device, created
 * on the first such call outside a stream capture and kept for the life of the
 * thread), forked from `stream` by an event after the compose backward and
 * joined back into `stream` by an event before the call returns: work queued
 * on `stream` afterwards sees all outputs, and a CUDA graph captured around the
 * call holds both branches. Under the kernel profiler the call stays on
 * `stream` alone.
 */
DORA_API dora_status_t dora_backward(const dora_desc_t* desc, int64_t T, const void* dy, const void* x, const void* W0,
                            const void* A, const void* B, const float* norm, const float* g, const void* su_save,
                            const void* pre_save, float* dm, void* dA, void* dB, void* dx, void* ws,
                            size_t ws_bytes, dora_stream_t stream);

/*
 * dora_backward_full -- the same gradients without the detach of the norm.
 *
 * DoRA notes appendix A eq. (A.1): through C the gradient of V'_n is
 * (m_n / C_n) (I - V'_n V'_n^T / C_n^2) grad W'_n. With
 * kappa_n = g_n dm_n / C_n (= m_n dm_n / C_n^2, dm as above) this is the
 * detached gradient minus kappa_n V'_n per row, V' = W0 + s B A, so
 *   dB_full = dB - s diag(kappa) (W0 A^T + s B A A^T)
 *   dA_full = dA - s (diag(kappa) B)^T W0 - s^2 (B^T diag(kappa) B) A
 * while dm and dx are unchanged (they do not pass through C). The dense V' is
 * never formed: the two extra products re-read W0 once each.
 * Arguments, layouts and errors as dora_backward; workspace from
 * dora_workspace_size(desc, T, DORA_OP_BACKWARD_FULL).
 */
DORA_API dora_status_t dora_backward_full(const dora_desc_t* desc, int64_t T, const void* dy, const void* x,
                                          const void* W0, const void* A, const void* B, const float* norm,
                                          const float* g, const void* su_save, const void* pre_save, float* dm,
                                          void* dA, void* dB, void* dx, void* ws, size_t ws_bytes,
                                          dora_stream_t stream);

/*
 * DVoRA -- DoRA notes section 3.5: the direction update of VeRA,
 * diag(b) B_shared diag(d) A_shared, with the random pair A_shared [r x d_in],
 * B_shared [d_out x r] shared and frozen, and only b [d_out], d [r] (and m)
 * trained. The layer is DoRA with A = A_shared and B = B' = diag(b) B_shared
 * diag(d): form B' with dora_vera_compose, run dora_norm / dora_forward /
 * dora_backward (or _full) / dora_merge on it unchanged, and turn the dB' they
 * return into the gradients of b and d with dora_vera_grad (dA is then not
 * needed: A_shared is frozen).
 *
 * dora_vera_compose: B_out[n][c] = b[n] B_shared[n][c] d[c], computed in fp32
 *   and rounded once to the desc dtype. B_shared, B_out [d_out x r] (dtype);
 *   b [d_out], d [r] fp32. No workspace.
 * dora_vera_grad: db[n] = sum_c dB[n][c] B_shared[n][c] d[c] and
 *   dd[c] = sum_n dB[n][c] b[n] B_shared[n][c], fp32, deterministic. dB is the
 *   gradient of B' [d_out x r] (dtype); db [d_out], dd [r] fp32 out.
 *   Workspace: dora_workspace_size(desc, 0, DORA_OP_VERA_GRAD).
 * Both read d_out, r and dtype from desc; desc->d_in and desc->s are not used.
 */
DORA_API dora_status_t dora_vera_compose(const dora_desc_t* desc, const void* B_shared, const float* b, const float* d,
                                         void* B_out, dora_stream_t stream);
DORA_API dora_status_t dora_vera_grad(const dora_desc_t* desc, const void* B_shared, const float* b, const float* d,
                                      const void* dB, float* db, float* dd, void* ws, size_t ws_bytes,
                                      dora_stream_t stream);

/*
 * dora_merge -- the merged deployment weight W' = diag(g) (W0 + s B A).
 *
 * DoRA notes Algorithm 1 steps 16-17 (merge after training: m (W0 + BA) / C
 * stored as one dense weight, so inference costs a plain linear layer).
 * In:  W0 [d_out x d_in], A [r x d_in], B [d_out x r] (dtype); g [d_out] fp32
 *      from dora_norm. Out: W_out [d_out x d_in] (dtype), rounded once.
 * W_out may be W0 itself (in-place merge): each output element is written by
 * the thread that read its W0 value, and nothing else reads W0.
 */
DORA_API dora_status_t dora_merge(const dora_desc_t* desc, const void* W0, const void* A, const void* B,
                                  const float* g, void* W_out, void* ws, size_t ws_bytes, dora_stream_t stream);

/*
 * dora_device_status -- synchronise `stream`, then read and clear the library's
 * device status word. *flags_out = 0 when every bounded wait in the kernels
 * finished in time; bit 0 set means some wait ran out (the results of the
 * calls since the last check are unreliable) and the call returns DORA_ETIMEOUT.
 */
DORA_API dora_status_t dora_device_status(dora_stream_t stream, unsigned int* flags_out);

/*
 * dora_selftest_timeout -- exercise the failure detection without a fault.
 * Launches one kernel on `stream` whose single thread waits, through the same
 * bounded wait the compute kernels use, on an mbarrier that nothing completes;
 * after limit_us microseconds (1 .. 1000000) the wait gives up, records the
 * timeout in the device status word and the kernel returns. The next
 * dora_device_status on that stream then reports bit 0 and DORA_ETIMEOUT, and
 * the context stays usable. scratch: one device word the kernel writes (1 =
 * the wait ran out). Nothing faults, traps or hangs.
 */
DORA_API dora_status_t dora_selftest_timeout(uint32_t limit_us, unsigned int* scratch, dora_stream_t stream);

/*
 * Kernel timing (benchmarks and tracing; not part of the compute path).
 * dora_profile_start(capacity) creates 2 * capacity CUDA events and, until
 * dora_profile_stop(), brackets each kernel the library launches with a pair of
 * them on the launch stream (as graph event-record nodes while the stream is
 * captured, so every graph replay re-times the same kernels). dora_profile_read
 * waits for the recorded events and fills up to `capacity` records in launch
 * order; `name` points to a static string naming the kernel. One host thread.
 */
typedef struct {
  const char* name;
  float ms;
} dora_profile_record_t;

DORA_API dora_status_t dora_profile_start(int capacity);
DORA_API dora_status_t dora_profile_stop(void);
DORA_API int dora_profile_count(void);
DORA_API dora_status_t dora_profile_read(dora_profile_record_t* out, int capacity, int* n_out);

/* Message for the last non-OK status returned on this thread ("" if none). */
DORA_API const char* dora_last_error(void);

/* Library version: major * 10000 + minor * 100 + patch. */
DORA_API int dora_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DORA_H_ */
