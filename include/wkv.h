/*
 * wkv.h -- C ABI of libwkv.so, a Blackwell (sm_100a) implementation of the RWKV
 * time-mixing WKV operator.
 *
 * The operation. "Linear attention without writing a CUDA kernel"
 * (anshulranjan.vercel.app), section "The recurrence", defines for each channel
 * c, with a per-channel decay w_c and bonus u_c,
 *
 *     wkv_t = ( sum_{i<t} e^{-(t-1-i)w + k_i} v_i + e^{u + k_t} v_t )
 *           / ( sum_{i<t} e^{-(t-1-i)w + k_i}     + e^{u + k_t}     )
 *
 * and the same section carries the two sums forward as a state
 * (numerator, denominator, max_exponent): the true pair is
 * N = num * e^{max_e}, D = den * e^{max_e}. One token first forms the output
 * from the state and the bonus-weighted current token, then decays the state by
 * e^{-w} and adds the current token (without the bonus). A state passed in is
 * used at the first token before any decay, exactly as the recurrence does.
 *
 * Conventions for every entry point:
 *   - All pointers are DEVICE pointers (memory the caller allocated with
 *     cudaMalloc or a caching allocator on the current device), unless a
 *     comment says otherwise. The caller owns every buffer; the library keeps
 *     no pointer after the call returns and allocates no device memory.
 *   - Layouts are dense and row-major: k, v, out are [B, T, C] with the channel
 *     axis fastest (element (b,t,c) at (b*T + t)*C + c); w, u are [C]; each of
 *     the three state arrays is [B, C] (or [S, C] for decode).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 *     default stream). The return value reports argument checks and launch
 *     errors only. Arguments are checked before anything is launched; a call
 *     that returns an error has launched nothing and written nothing.
 *   - Inputs must be finite. The empty state is (0, 0, -inf); any state with
 *     den <= 0 or max_e = -inf is treated as empty.
 *   - out must not overlap k, v, w, u or the state arrays.
 *   - Results are bitwise reproducible for fixed shapes, dtypes, options and
 *     device.
 */
#ifndef WKV_H
#define WKV_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define WKV_API __attribute__((visibility("default")))
#else
#define WKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    WKV_OK = 0,
    WKV_ERR_INVALID_ARG = 1,        /* negative size, NULL pointer, bad option value */
    WKV_ERR_UNSUPPORTED_DTYPE = 2,  /* dtype combination not in the list below */
    WKV_ERR_MISALIGNED = 3,         /* workspace not 256-byte aligned (misaligned k, v, out: slower path, no error) */
    WKV_ERR_WORKSPACE_TOO_SMALL = 4,
    WKV_ERR_CUDA = 5,               /* a CUDA runtime call failed (no device, launch error) */
    WKV_ERR_WAIT_TIMEOUT = 6,       /* device side: a bounded wait gave up (see wkv_query_status) */
    WKV_ERR_BOUNDS = 7              /* device side, the bounds-checked build (libwkv_debug.so, compiled
                                       with -DWKV_DEBUG) only: an index outside its array was caught and
                                       the access skipped (see wkv_query_status) */
} wkv_status;

typedef enum { WKV_F32 = 0, WKV_BF16 = 1 } wkv_dtype;

/* State read by a call: three fp32 arrays (num, den, max_e), each [B, C]. */
typedef struct {
    const float *num;
    const float *den;
    const float *max_e;
} wkv_cstate;

/* State written by a call: three fp32 arrays, each [B, C]. They may be the
 * very same arrays as a wkv_cstate of the same call (in-place update). */
typedef struct {
    float *num;
    float *den;
    float *max_e;
} wkv_state;

/*
 * Dispatch and test controls for wkv_forward. Pass NULL for the defaults; a
 * zero-filled struct also means "defaults".
 *   kernel          0 = choose by shape: sequential for many channels
 *                   (B*C >= 65536) or short sequences (T <= 64); otherwise the
 *                   cluster scan above 2^24 elements of k (B*T*C; k and v
 *                   larger than L2), else the three-launch scan,
 *                   1 = sequential-over-T kernel,
 *                   2 = chunked scan in one launch (look-back between CTAs),
 *                   3 = chunked scan in three launches (chunk totals, their
 *                   scan, then the replay; k and v are read twice, from L2
 *                   the second time for inputs that fit there),
 *                   4 = chunked scan in one launch of persistent CTAs that
 *                   pipeline their tiles (look-back of one tile overlapped
 *                   with the next tile's fold and later tiles' copies),
 *                   5 = chunked scan in thread-block clusters: a cluster of
 *                   up to 2 CTAs takes a segment of 2 x cta_warps x span
 *                   tokens of one (batch row, 32 channels); each warp streams
 *                   its span through its own TMA ring twice (fold, then
 *                   replay), the CTAs exchange their totals through
 *                   distributed shared memory, and the segments of a channel
 *                   group chain through the inclusive prefix each publishes
 *                   for the next; one launch, k and v read once from memory
 *                   (the replay re-reads them from L2)
 *   chunk_len       tokens per chunk for the chunked kernels (0 = choose: 32
 *                   or 64 for the three-launch scan, 128 otherwise; or 32, 64,
 *                   128)
 *   lookback_group  G: the chunked kernel publishes a running prefix every G
 *                   chunks and each chunk combines at most G-1 chunk totals
 *                   after the last one (0 = choose; otherwise 1..1024)
 *   wait_timeout_ns limit of every device-side wait (0 = 1 second)
 *   span            tokens per warp in a chunk-scan tile, 8 or 16 (0 = choose);
 *                   chunk_len / span warps share a tile (at most 8 for the
 *                   pipelined scan, so chunk_len 128 needs span 16 there);
 *                   the cluster scan (kernel 5) takes 32 or 64 (0 = 64)
 *   seq_threads     threads per CTA of the sequential kernel and of the
 *                   three-launch scan's replay pass: 32, 64 or 128 (0 =
 *                   choose: 32); each thread carries seq_vec channels in the
 *                   sequential kernel, one in the replay pass
 *   scan_segments   three-launch scan (kernel 3): segments per channel in the
 *                   scan of the chunk totals: 0 = choose, or 1, 4, 16, 64
 *   seq_vec         channels per thread of the sequential kernel: 1 or 2
 *                   (0 = choose: 1 below 151552 channels B*C, else 2)
 *   replay_chunks   three-launch scan (kernel 3): consecutive chunks that
 *                   one replay warp walks (0 = choose; or 1, 2, 4)
 *   cta_warps       cluster scan (kernel 5): warps (spans) per CTA, 4 or 8
 *                   (0 = 8)
 *   stages          shared-memory ring stages of the pipelined scan
 *                   (kernel 4): 0 = choose, otherwise 2..8 (must fit in one
 *                   CTA's shared memory, else WKV_ERR_INVALID_ARG at launch)
 *   inject_enable, inject_unpublished_tile
 *                   tests of the bounded waits only: with inject_enable = 1,
 *                   chunk-scan tile number inject_unpublished_tile (in the
 *                   cluster scan: the cluster with that ticket) computes
 *                   but never publishes its result, so the tiles that wait for
 *                   it reach their wait limit, carry on, and the call reports
 *                   WKV_ERR_WAIT_TIMEOUT through wkv_query_status. 0 = off.
 */
typedef struct {
    int32_t kernel;
    int32_t chunk_len;
    int32_t lookback_group;
    int32_t inject_enable;
    int64_t wait_timeout_ns;
    int64_t inject_unpublished_tile;
    int32_t span;
    int32_t seq_threads;
    int32_t scan_segments;
    int32_t stages;
    int32_t seq_vec;
    int32_t replay_chunks;
    int32_t cta_warps;
} wkv_options;

/*
 * Bytes of workspace that wkv_forward needs for these sizes and options.
 * Host-only; touches no device. The workspace must be zero-filled before its
 * first use; the library leaves it ready for the next call. One workspace must
 * not be used by two calls that may run at the same time.
 */
WKV_API size_t wkv_forward_workspace_size(int64_t B, int64_t T, int64_t C, const wkv_options *opts);

/*
 * The kernel (1..4, numbered as wkv_options.kernel) that wkv_forward launches
 * for these sizes, input dtype and options, for k and v whose base addresses
 * are 16-byte aligned; 0 for invalid arguments. Host-only; touches no device.
 */
WKV_API int32_t wkv_forward_kernel(int64_t B, int64_t T, int64_t C, wkv_dtype kv_dtype, const wkv_options *opts);

/*
 * How many kernels one wkv_forward call launches for these sizes, input dtype
 * and options (16-byte aligned k and v, T > 0); 0 for invalid arguments or
 * when there is nothing to compute. Host-only; touches no device.
 */
WKV_API int32_t wkv_forward_launches(int64_t B, int64_t T, int64_t C, wkv_dtype kv_dtype, const wkv_options *opts);

/*
 * Sequence forward: for every (b, c), run the recurrence over t = 0..T-1,
 * starting from state_in (NULL = the empty state), write wkv_t to out and the
 * state after the last token to state_out (NULL = not written).
 *
 *   k, v       [B, T, C], element type kv_dtype
 *   w, u       [C] fp32: decay (the state is multiplied by e^{-w} per token)
 *              and bonus of the current token
 *   out        [B, T, C], element type out_dtype
 *   state_in   NULL, or three fp32 [B, C] arrays
 *   state_out  NULL, or three fp32 [B, C] arrays; may alias state_in
 *   workspace  device buffer of at least wkv_forward_workspace_size() bytes,
 *              zero-filled before its first use; it also carries the
 *              device-side status word read by wkv_query_status
 *   stream     cudaStream_t
 *   opts       NULL for defaults
 *
 * Supported dtypes: (kv F32, out F32), (kv BF16, out BF16), (kv BF16, out F32).
 * Sizes: B, T, C >= 0, T < 2^24, B*T*C < 2^62. T = 0 copies state_in to
 * state_out (or writes the empty state when state_in is NULL).
 * The state is always fp32 and the arithmetic is fp32.
 */
WKV_API wkv_status wkv_forward(int64_t B, int64_t T, int64_t C,
                       const void *k, const void *v, wkv_dtype kv_dtype,
                       const float *w, const float *u,
                       void *out, wkv_dtype out_dtype,
                       const wkv_cstate *state_in, const wkv_state *state_out,
                       void *workspace, size_t workspace_bytes,
                       void *stream, const wkv_options *opts);

/*
 * Sequence forward over HOST-resident k, v and out ([B, T, C] in host
 * memory; page-locked for the copies to overlap), for inputs that live on the
 * host: the sequence is cut into segments of seg_tokens tokens (0 = choose:
 * about 64 MB of k and v per segment). Segment s is copied to the device on
 * streams of the library's own (k and v on one each), computed by wkv_forward
 * on `stream` from the state after segment s-1, and its outputs copied back
 * on a third library stream; two segments are in flight, so the copies in,
 * the compute and the copies back of neighbouring segments run side by side.
 *   w, u, state_in, state_out  device arrays, as for wkv_forward
 *   dev_buffer  device buffer of at least wkv_forward_host_buffer_size()
 *               bytes, 256-byte aligned and zero-filled before its first use
 *               (two segments of k, v and out, the carried state, and the
 *               forward's workspace); owned by the caller
 * Returns once the work is queued; it has all completed when `stream` has
 * (the library's streams fork from `stream` at the call and join it before
 * its end, also under stream capture once a first call on the device has
 * created them outside of capture). The result equals wkv_forward's with the
 * sequence split at the segment boundaries (the state handed from segment to
 * segment as wkv_forward's state out). Errors as wkv_forward's, and
 * WKV_ERR_WORKSPACE_TOO_SMALL for a dev_buffer below the size.
 */
WKV_API size_t wkv_forward_host_buffer_size(int64_t B, int64_t T, int64_t C, wkv_dtype kv_dtype,
                                            wkv_dtype out_dtype, int64_t seg_tokens);
WKV_API wkv_status wkv_forward_host(int64_t B, int64_t T, int64_t C,
                            const void *k_host, const void *v_host, wkv_dtype kv_dtype,
                            const float *w, const float *u,
                            void *out_host, wkv_dtype out_dtype,
                            const wkv_cstate *state_in, const wkv_state *state_out,
                            void *dev_buffer, size_t dev_bytes, int64_t seg_tokens,
                            void *stream);

/*
 * Two optional inputs of the RWKV-v6 time-mixing block ("RWKV-v6
 * Architecture: Attention-Free Linear Transformers"), for wkv_forward_ext and
 * wkv_step_ext:
 *   w_t  NULL, or fp32 decays of every token ([B, T, C] for a forward, [S, C]
 *        for a decode step), in place of w: token t's advance multiplies the
 *        state by e^{-w_t} (section "2. Dynamic Data-Dependent Decay"; the
 *        page's multiplicative factor exp(-exp(.)) is e^{-w_t} here). An
 *        earlier token i then reaches token t with the exponent
 *        k_i - (w_{i+1} + ... + w_{t-1}).
 *   r    NULL, or the receptance, same shape and element type as k: every
 *        output is gated, out = sigmoid(r) * wkv (the readout of section
 *        "3. Matrix-Valued Hidden State"). The state is not gated.
 */
typedef struct {
    const float *w_t;
    const void *r;
} wkv_ext;

/*
 * wkv_forward with the optional inputs of wkv_ext (ext = NULL, or both of its
 * pointers NULL, is exactly wkv_forward). With w_t, the w argument is not read
 * and may be NULL. Kernels: r works with every kernel; w_t with the
 * sequential kernel (1), the three-launch scan (3) and the cluster scan (5);
 * an explicit kernel 2 or 4 with w_t is WKV_ERR_INVALID_ARG, and the automatic
 * choice never takes them with w_t.
 */
WKV_API wkv_status wkv_forward_ext(int64_t B, int64_t T, int64_t C,
                           const void *k, const void *v, wkv_dtype kv_dtype,
                           const float *w, const float *u,
                           void *out, wkv_dtype out_dtype,
                           const wkv_cstate *state_in, const wkv_state *state_out,
                           void *workspace, size_t workspace_bytes,
                           void *stream, const wkv_options *opts, const wkv_ext *ext);

/*
 * Batched one-token decode (the constant-cost step of the recurrence): S
 * independent streams of C channels each take one token.
 *
 *   k, v       [S, C], element type kv_dtype
 *   w, u       [C] fp32
 *   out        [S, C], element type out_dtype
 *   state_in   required: three fp32 [S, C] arrays (the empty state is allowed)
 *   state_out  required: three fp32 [S, C] arrays; may alias state_in (in place)
 *   stream     cudaStream_t
 *
 * Needs no workspace and has no device-side waits. Capture-safe: no host
 * synchronisation and no allocation.
 */
WKV_API wkv_status wkv_step(int64_t S, int64_t C,
                    const void *k, const void *v, wkv_dtype kv_dtype,
                    const float *w, const float *u,
                    void *out, wkv_dtype out_dtype,
                    const wkv_cstate *state_in, const wkv_state *state_out,
                    void *stream);

/*
 * wkv_step with the optional inputs of wkv_ext: w_t [S, C] (this token's decay
 * for every stream, in place of w, which may then be NULL) and r [S, C]
 * (element type kv_dtype). ext = NULL is exactly wkv_step.
 */
WKV_API wkv_status wkv_step_ext(int64_t S, int64_t C,
                        const void *k, const void *v, wkv_dtype kv_dtype,
                        const float *w, const float *u,
                        void *out, wkv_dtype out_dtype,
                        const wkv_cstate *state_in, const wkv_state *state_out,
                        void *stream, const wkv_ext *ext);

/*
 * Backward of wkv_forward (per-channel w, no w_t or r): the gradients of a
 * loss L given gout = dL/d wkv for every output, with no loss term on the
 * final state. The chain rule through the step function of "The recurrence"
 * run backwards in time; the pages' claim that the recurrence trains like a
 * transformer ("What held up": it trains; "RWKV-v6 Architecture", "Key
 * Mechanics: Architectural Duality", time-parallel mode) is what makes it
 * part of the operator:
 *     dv_t = g_t e^{u+k_t}/Z_t + e^{k_t} dN_{t+1}
 *     dk_t = g_t e^{u+k_t}(v_t - wkv_t)/Z_t + e^{k_t}(v_t dN_{t+1} + dD_{t+1})
 *     du   = sum_{b,t} g_t e^{u+k_t}(v_t - wkv_t)/Z_t
 *     dw   = -sum_{b,t} e^{-w}(N_t dN_{t+1} + D_t dD_{t+1})
 * with (N_t, D_t) the state pair before token t, Z_t = D_t + e^{u+k_t}, and
 * dN_t = g_t/Z_t + e^{-w} dN_{t+1}, dD_t = -g_t wkv_t/Z_t + e^{-w} dD_{t+1}.
 *
 *   k, v       [B, T, C], element type kv_dtype, base addresses 16-byte
 *              aligned and C * element size a multiple of 16 bytes (else
 *              WKV_ERR_MISALIGNED)
 *   w, u       [C] fp32;  state_in  NULL or three fp32 [B, C] (as wkv_forward)
 *   gout       [B, T, C] fp32, base address 16-byte aligned
 *   dk, dv     [B, T, C] fp32 (written)
 *   dw, du     [C] fp32 (written; summed over the batch rows)
 *   dstate_in  NULL, or three fp32 [B, C] arrays receiving dL/dnum, dL/dden,
 *              dL/dmax_e of state_in (zeros where it was empty or absent)
 *   workspace  at least wkv_backward_workspace_size(B, T, C) bytes, 256-byte
 *              aligned; no zero-fill needed (every byte read is written first)
 * Results are bitwise reproducible. Launches six kernels (four when T <= 32).
 */
WKV_API size_t wkv_backward_workspace_size(int64_t B, int64_t T, int64_t C);
WKV_API wkv_status wkv_backward(int64_t B, int64_t T, int64_t C,
                        const void *k, const void *v, wkv_dtype kv_dtype,
                        const float *w, const float *u,
                        const wkv_cstate *state_in, const float *gout,
                        float *dk, float *dv, float *dw, float *du,
                        const wkv_state *dstate_in,
                        void *workspace, size_t workspace_bytes, void *stream);

/*
 * The RWKV-v6 matrix-valued state ("RWKV-v6 Architecture: Attention-Free
 * Linear Transformers", section "3. Matrix-Valued Hidden State"): per head a
 * D x D state S, and for every token
 *     S_t = diag(w_t) S_{t-1} + k_t v_t^T,     y_t = sigmoid(r_t) * (S_t k_t)
 * (row i of S decays by w_t[i]; the readout multiplies the updated state by
 * k_t, as the page writes it). A different operator from wkv_forward: no
 * denominator and no max exponent.
 *
 *   r, k, v    [B, T, H, D], element type kv_dtype
 *   w          [B, T, H, D] fp32: the decay factor itself, in [0, 1] (the
 *              page's exp(-exp(.)) of a projection)
 *   y          [B, T, H, D], element type y_dtype ((F32, F32), (BF16, BF16)
 *              or (BF16, F32))
 *   state_in   NULL (zero state) or [B, H, D, D] fp32, S[b][h][i][j] with i
 *              the row (key) index; state_out NULL or the same shape, may
 *              alias state_in
 *   D          32, 64 or 128
 *   workspace  at least 256 bytes, 256-byte aligned, zero-filled before its
 *              first use: its status word reports device-side wait timeouts
 *              (wkv_query_status)
 * r, w, k, v must be 16-byte aligned (WKV_ERR_MISALIGNED otherwise). The
 * arithmetic and the state are fp32; results are bitwise reproducible. A
 * decode step is a call with T = 1.
 */
WKV_API wkv_status wkv_v6_forward(int64_t B, int64_t T, int64_t H, int64_t D,
                        const void *r, const float *w, const void *k, const void *v, wkv_dtype kv_dtype,
                        void *y, wkv_dtype y_dtype,
                        const float *state_in, float *state_out,
                        void *workspace, size_t workspace_bytes, void *stream);

/*
 * wkv_forward without a caller-provided workspace. The pages have no
 * counterpart to this entry point; it exists for callers that cannot allocate
 * device memory themselves: hosts that hand a plug-in only its input and
 * output buffers while their own pool owns the rest of the GPU, and code with
 * hard latency limits, where cudaMalloc's implicit synchronisation of the
 * device is not acceptable.
 *
 * Same arguments and results as wkv_forward with default options, except that
 * the scratch memory lives in a fixed array of WKV_NOALLOC_SCRATCH_BYTES bytes
 * inside the library (every GPU that loads the library holds it until the
 * process exits). The call allocates nothing.
 *   - Shapes whose scratch need (wkv_forward_workspace_size(B, T, C, NULL))
 *     exceeds WKV_NOALLOC_SCRATCH_BYTES are rejected with
 *     WKV_ERR_WORKSPACE_TOO_SMALL before anything is launched.
 *   - The first call on a device looks up the array's device address (with
 *     that device current); make that first call before any stream capture.
 *   - Every call zeroes the array's counters and flags on `stream` before its
 *     kernel runs. All calls share the one array: two calls that may overlap on
 *     the GPU (different streams, or different host threads) race and give
 *     wrong results; serialise them.
 *   - Device-side wait timeouts are not reported through this entry point
 *     (there is no workspace to query); the waits still end at their limit.
 */
#define WKV_NOALLOC_SCRATCH_BYTES (16u << 20)
WKV_API wkv_status wkv_forward_noalloc(int64_t B, int64_t T, int64_t C,
                               const void *k, const void *v, wkv_dtype kv_dtype,
                               const float *w, const float *u,
                               void *out, wkv_dtype out_dtype,
                               const wkv_cstate *state_in, const wkv_state *state_out,
                               void *stream);

/*
 * Synchronises `stream`, then reads and clears the device-side status word in
 * `workspace` (a wkv_forward, wkv_backward or wkv_v6_forward workspace).
 * Returns WKV_OK, WKV_ERR_BOUNDS (bounds-checked build only), WKV_ERR_WAIT_TIMEOUT
 * if a device-side wait of an earlier call gave up (its outputs are then not
 * valid), or WKV_ERR_CUDA if the synchronisation itself failed.
 */
WKV_API wkv_status wkv_query_status(void *workspace, void *stream);

/* Static English text for a status code. Host-only. */
WKV_API const char *wkv_status_string(wkv_status status);

/* Library version as 10000*major + 100*minor + patch. Host-only. */
WKV_API int32_t wkv_version(void);

/*
 * Name of the last CUDA runtime error that made a call of this library in the
 * calling thread return WKV_ERR_CUDA ("cudaSuccess" if none has). Static
 * text; host-only; the record is not cleared by reading it.
 */
WKV_API const char *wkv_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* WKV_H */
