/*
 * sa_sketch.h -- C ABI of libsa_sketch.so: Sketch Attention (SA) forward and
 * backward on B200 (sm_100a).
 *
 * What SA computes. The sources are the "100,000 videos in your pocket" blog,
 * section "1. Sketch Attention compresses the history", and the evolve.pub review
 * of arXiv 2609.08443, "Summary" and its FAQ on how SA differs from standard
 * attention. Per user u, with history tokens t in [offsets[u], offsets[u+1]):
 *
 *   K = X W_k,  V = X W_v                       learnable prototypes P (k x d)
 *   s_jt = P_j . K_t / sqrt(d)                  prototypes score every token
 *   A_jt = exp(s_jt) / sum_i exp(s_it)          normalised across prototypes:
 *                                               each token spreads unit mass
 *   mass_j   = sum_t A_jt
 *   sketch_j = (sum_t A_jt V_t) / mass_j        fixed k x d, target-agnostic
 *
 * The pages give no equations. The projections, the 1/sqrt(d) scale, the softmax
 * normaliser and the mass-weighted mean are the plainest reading of them.
 * Several users of different lengths are processed in one call as a ragged batch.
 * The batch is described by an offsets array (blog, "3. The system makes it cheap
 * enough to matter": a fused kernel under ragged batches, with multi-request
 * user-level batching).
 *
 * Conventions for every entry point:
 *  - All pointer arguments are DEVICE pointers unless stated otherwise. All
 *    matrices are dense and row-major. The caller allocates and owns every
 *    buffer; these calls allocate nothing.
 *  - Calls are asynchronous and stream-ordered on `stream`. A cudaStream_t is
 *    passed as void*; NULL means the legacy default stream.
 *  - Argument errors are detected on the host. They return a non-zero status
 *    before anything is launched.
 *  - Some errors are only visible on the device: offsets that are not
 *    non-decreasing, offsets[0] != 0, offsets[R] != n_total, or a bounded wait
 *    inside a kernel that gave up. These are latched in a status word inside the
 *    workspace. sa_sketch_get_device_status() reads that word. When it is set,
 *    the outputs of that call are unspecified. The kernels never trap.
 *  - `workspace` must be at least sa_sketch_workspace_size(...) bytes, 256-byte
 *    aligned, and not used by another call in flight. Its contents need no
 *    initialisation; each call initialises what it uses.
 */
#ifndef SA_SKETCH_H
#define SA_SKETCH_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Element type of X, P, W_k and W_v (every output is fp32). */
typedef enum { SA_F32 = 0, SA_BF16 = 1 } sa_dtype;

typedef enum {
  SA_OK = 0,
  SA_ERR_INVALID_ARG = 1,   /* null pointer, negative size, misaligned pointer   */
  SA_ERR_UNSUPPORTED = 2,   /* shape outside what the kernels implement          */
  SA_ERR_WORKSPACE = 3,     /* workspace null, misaligned or too small           */
  SA_ERR_CUDA = 4,          /* a CUDA runtime call failed (launch, copy, ...)     */
  SA_ERR_TIMEOUT = 5,       /* device: a bounded wait inside a kernel gave up    */
  SA_ERR_BAD_OFFSETS = 6,   /* device: offsets not a valid ragged partition      */
  SA_ERR_NO_DEVICE = 7      /* no sm_100 device current                          */
} sa_status;

/* Limits. d must be 64 or 128. k may be 1..2048 for fp32 and bf16 alike; bf16
 * runs on tcgen05 tensor cores in slices of 128 prototypes, with k padded up to a
 * multiple of 128 inside the kernel. R may be 0..SA_MAX_USERS and n_total may be
 * 0..2^31-1. */
#define SA_MAX_K 2048
#define SA_MAX_USERS (1 << 20)

/*
 * Bytes of device workspace that sa_sketch_forward (backward = 0) or
 * sa_sketch_backward (backward = 1) needs for these sizes on the current device.
 * The plan depends on the device's SM count, so query it with the device current
 * that will run the call. Returns 0 if the sizes are unsupported.
 * For the bf16 forward this is the plan with the helper grid (sa_sketch_forward_grid),
 * whose helper CTAs add H segments of k_pad x (d + 1) floats. Given less than that but
 * at least the plan without them, sa_sketch_forward runs the clustered grid alone
 * (slower; same results to rounding).
 */
size_t sa_sketch_workspace_size(int R, int64_t n_total, int k, int d, sa_dtype dt,
                                int backward);

/*
 * Forward. Sources: blog section "1. Sketch Attention compresses the history" and
 * review "Summary" (prototype scoring, prototype-wise normalisation, k x d sketch).
 *
 *   X       [n_total, d]  dt    history tokens of all users, concatenated
 *   offsets [R + 1]       int64 offsets[0] = 0, non-decreasing, offsets[R] = n_total
 *   P       [k, d]        dt    prototypes, shared by all users
 *   Wk, Wv  [d, d]        dt    key and value projections (K = X Wk, V = X Wv)
 * Outputs (fp32, overwritten):
 *   sketch  [R, k, d]     mass-weighted mean of values per prototype
 *   mass    [R, k]        sum over the user's tokens of A_jt
 *   lse     [n_total]     per-token log-sum-exp of the scores (natural log);
 *                         nullable. Needed by the backward.
 *   xsketch [R, k, d]     sum_t A_jt X_t (un-normalised, before W_v); nullable.
 *                         Needed by the backward.
 * A user with no tokens gets sketch = 0 and mass = 0. Results are deterministic:
 * two calls on the same inputs give bitwise-equal outputs.
 * Precision of the bf16 path: the scores use P' = P Wk^T / sqrt(d) rounded to bf16 and
 * A is rounded to bf16 before it meets X; accumulation is fp32. When k is a multiple of
 * 128, sketch = (U / mass) Wv runs on the tensor cores with U / mass split into two bf16
 * parts (about 16 significant bits), else in fp32 on the CUDA cores.
 * Pointers must be 16-byte aligned.
 */
int sa_sketch_forward(const void* X, const int64_t* offsets, int R, int64_t n_total, int d,
                      const void* P, int k, const void* Wk, const void* Wv, sa_dtype dt,
                      float* sketch, float* mass, float* lse, float* xsketch,
                      void* workspace, size_t ws_bytes, void* stream);

/*
 * Backward. SA is differentiable, so the ranking loss's gradient flows back
 * through the compression (blog, "1. Sketch Attention compresses the history").
 * Given G = dL/dsketch and optional Gm = dL/dmass, this writes the gradients with
 * respect to X, P, Wk and Wv.
 *
 *   X, offsets, P, Wk, Wv, dt   as passed to the forward
 *   sketch, mass, xsketch       fp32 outputs of that forward (required)
 *   lse                         the forward's lse for the same inputs, nullable. The
 *                               bf16 path uses it when given (else it recomputes it, one
 *                               more k x n x d contraction); the fp32 path recomputes
 *                               the per-token statistics and does not read it
 *   dsketch [R, k, d] fp32      G
 *   dmass   [R, k]    fp32      Gm; nullable (NULL means zero)
 * Outputs (fp32, overwritten, not accumulated into):
 *   dX  [n_total, d]
 *   dP  [k, d], dWk [d, d], dWv [d, d]   summed over all users
 * bf16 inputs run on the tensor cores: the token x prototype intermediates (the softmax
 * A and its gradient dS, bf16: 4 bytes per token and prototype) live in the workspace,
 * which sa_sketch_workspace_size(..., backward = 1) sizes accordingly (about 8 GB at
 * 1.8 M tokens and k = 1024). fp32 inputs run on CUDA cores with a small workspace.
 */
int sa_sketch_backward(const void* X, const int64_t* offsets, int R, int64_t n_total, int d,
                       const void* P, int k, const void* Wk, const void* Wv, sa_dtype dt,
                       const float* sketch, const float* mass, const float* lse,
                       const float* xsketch, const float* dsketch, const float* dmass,
                       float* dX, float* dP, float* dWk, float* dWv,
                       void* workspace, size_t ws_bytes, void* stream);

/*
 * Forward from HOST inputs to HOST outputs, with the copies overlapped with the compute.
 * Same computation as sa_sketch_forward (blog "1. Sketch Attention compresses the
 * history"); users are independent, and the batch is ragged (blog "3. The system makes it
 * cheap enough to matter": multi-request user-level batching), so the call cuts the users
 * into at most `parts` consecutive parts of about equal token count
 * (sa_sketch_host_parts) and pipelines them: part p's X is copied to the device on
 * `h2d_stream` while part p - 1's forward runs on `stream`, and part p's sketch and mass
 * are copied back on `d2h_stream` as soon as its forward has finished.
 *
 *   X_host       [n_total, d] dt, HOST       history tokens of all users
 *   offsets_host [R + 1] int64, HOST         offsets[0] = 0, non-decreasing,
 *                                            offsets[R] = n_total (checked on the host)
 *   P, Wk, Wv    dt, DEVICE                  as for sa_sketch_forward
 *   sketch_host  [R, k, d] fp32, HOST        output (overwritten)
 *   mass_host    [R, k] fp32, HOST           output (overwritten)
 *   device_buffer, device_bytes              DEVICE scratch of at least
 *                sa_sketch_forward_host_buffer_size(...) bytes, 256-byte aligned: the
 *                device copy of X and offsets, the device sketch and mass, and the
 *                forward's workspace. Not shared with another call in flight.
 *   parts        1..64 (use 1 when k is not a multiple of 4)
 *   stream, h2d_stream, d2h_stream           three cudaStream_t (as void*); the two copy
 *                streams should be distinct from `stream` and from each other for the
 *                copies to overlap (the default stream serialises everything)
 * The call only enqueues work. The outputs are complete once `stream` has reached the end
 * of this call's work (synchronise it, or record an event on it). X_host and offsets_host
 * must stay unchanged until then. For the copies to run asynchronously the four host
 * buffers must be page-locked (cudaHostAlloc or cudaHostRegister); pageable buffers give
 * correct results but serialise the copies with the host. It creates and releases a few
 * CUDA events per call and allocates no memory. Returns SA_OK, the argument codes of
 * sa_sketch_forward, SA_ERR_BAD_OFFSETS (offsets_host invalid), SA_ERR_WORKSPACE or
 * SA_ERR_CUDA. Device-side errors are latched in the workspace inside device_buffer, at
 * offset 0 of the workspace region; read them with sa_sketch_forward_host_status.
 */
size_t sa_sketch_forward_host_buffer_size(int R, int64_t n_total, int k, int d, sa_dtype dt,
                                          int parts);
int sa_sketch_forward_host(const void* X_host, const int64_t* offsets_host, int R,
                           int64_t n_total, int d, const void* P, int k, const void* Wk,
                           const void* Wv, sa_dtype dt, float* sketch_host, float* mass_host,
                           void* device_buffer, size_t device_bytes, int parts, void* stream,
                           void* h2d_stream, void* d2h_stream);

/*
 * Device status word of the last sa_sketch_forward_host call that used `device_buffer`
 * with these sizes (synchronises `stream`); the same codes as sa_sketch_get_device_status.
 */
int sa_sketch_forward_host_status(const void* device_buffer, int R, int64_t n_total, int k,
                                  int d, sa_dtype dt, int parts, void* stream);

/*
 * The cut that sa_sketch_forward_host uses: users [0, R) into at most `parts` consecutive
 * parts of about equal token count. Cut c ends a part at the first user whose tokens
 * reach c / parts of the total; a cut that would leave a part without tokens is dropped,
 * and users without tokens at the end join the last part, so every part but a lone one
 * holds tokens and no user is split. Writes the part boundaries to bounds[0..np] (HOST,
 * room for parts + 1 ints; bounds[0] = 0, bounds[np] = R) and returns np (0 when R = 0),
 * or -SA_ERR_INVALID_ARG if the offsets are not a valid ragged partition. Host only.
 */
int sa_sketch_host_parts(const int64_t* offsets_host, int R, int parts, int* bounds);

/*
 * Epilogue for a user whose tokens were split across calls (for example across GPUs,
 * one part per rank). The forward's accumulation is a plain sum over tokens, so the
 * parts' xsketch and mass outputs add up to the whole user's (the sketch's definition
 * as a mass-weighted mean of V over tokens; blog "1. Sketch Attention compresses the
 * history"). After the caller has summed them (an all-reduce), this writes
 *   sketch_j = (xsketch_j Wv) / mass_j   (0 where mass_j = 0)
 * exactly as the forward's own last step does.
 *
 *   xsketch [R, k, d] fp32, device   sums of the parts' xsketch outputs
 *   mass    [R, k]    fp32, device   sums of the parts' mass outputs
 *   Wv      [d, d]    dt, device     as passed to the forward
 *   sketch  [R, k, d] fp32, device   output (overwritten)
 * d in {64, 128}; k >= 1. Pointers 16-byte aligned. Needs no workspace, allocates
 * nothing, enqueues one kernel on `stream` and does not synchronise. Returns SA_OK,
 * SA_ERR_INVALID_ARG, SA_ERR_UNSUPPORTED or SA_ERR_CUDA.
 */
int sa_sketch_combine(const float* xsketch, const float* mass, int R, int k, int d,
                      const void* Wv, sa_dtype dt, float* sketch, void* stream);

/*
 * Forward without a workspace, for callers that cannot allocate device memory (for
 * example a serving process whose allocator reserved all of its memory at start-up and
 * forbids new allocations, or code running where cudaMalloc may not be called). The
 * pages describe no such interface; it has no counterpart in the paper.
 *
 * Same arguments, results and conventions as sa_sketch_forward, minus the workspace.
 * The scratch space is one device array of SA_NOALLOC_SCRATCH_BYTES per GPU, held until
 * the process exits. It is reserved when the CUDA module that holds it loads on that GPU:
 * at the first use of the library's kernels under lazy module loading (the default), but
 * already when the context is created under CUDA_MODULE_LOADING=EAGER, in which case every
 * process that loads this library holds it on every GPU it uses, whether or not it calls
 * this entry point.
 *  - The first call on each device looks up the array's device address (set-up, with
 *    that device current). Make that first call before any stream capture begins.
 *  - Every call on a device shares the one array: calls whose work overlaps on the GPU
 *    (different streams, or different host threads) race and give wrong results.
 *    Serialise them, for instance on one stream.
 *  - Sizes whose plan needs more than SA_NOALLOC_SCRATCH_BYTES are rejected with
 *    SA_ERR_WORKSPACE before anything is launched (at k = 1024, d = 128 on a B200 about 24 users).
 *    When the scratch holds the plan without the helper grid but not with it, the call
 *    runs the clustered grid alone (see sa_sketch_forward's workspace).
 *  - It calls no cudaMalloc, cudaFree or allocating library routine.
 *  - device_status: nullable HOST pointer. When given, the call waits for `stream` and
 *    stores the device status word there (SA_OK, SA_ERR_BAD_OFFSETS, SA_ERR_TIMEOUT), since
 *    the caller cannot name the scratch array in sa_sketch_get_device_status. If that read
 *    fails (for example a stream in capture, or an earlier asynchronous CUDA error), the
 *    call returns SA_ERR_CUDA and leaves *device_status unchanged. Pass NULL while a stream
 *    capture is active.
 *  - Argument errors give the same codes as sa_sketch_forward.
 */
#define SA_NOALLOC_SCRATCH_BYTES (32u << 20)
int sa_sketch_forward_noalloc(const void* X, const int64_t* offsets, int R, int64_t n_total,
                              int d, const void* P, int k, const void* Wk, const void* Wv,
                              sa_dtype dt, float* sketch, float* mass, float* lse,
                              float* xsketch, int* device_status, void* stream);

/*
 * Launch shape of the bf16 forward on the current device. The persistent grid holds
 * *clusters clusters of *cluster_size CTAs (one CTA per 128 prototypes); when those
 * leave SMs free, *helpers helper CTAs (one per free SM, no cluster) run beside them and
 * take *helper_share / 1024 of the tiles. With T 128-token tiles in the batch (users'
 * tiles concatenated), Th = floor(T * helper_share / 1024) (0 when that is less than
 * 32 * helpers: the helpers take work only in full 32-tile chunks) and T1 = T - Th, cluster g
 * walks tiles [g T1 / clusters, (g + 1) T1 / clusters) and helper b walks
 * [T1 + b Th / helpers, T1 + (b + 1) Th / helpers). A user whose tiles straddle one of
 * those bounds is accumulated by two of them and summed in the finalize. For fp32
 * inputs (CUDA-core path) all four are set to 0. `helpers` and `helper_share` may be
 * null. Returns SA_OK, or the argument codes of sa_sketch_forward.
 */
int sa_sketch_forward_grid(int k, int d, sa_dtype dt, int* clusters, int* cluster_size,
                           int* helpers, int* helper_share);

/*
 * Reads the device status word that the last call using `workspace` left behind.
 * It synchronises `stream` and returns SA_OK, SA_ERR_BAD_OFFSETS or SA_ERR_TIMEOUT,
 * or SA_ERR_CUDA if the copy itself failed. The word is cleared at the start of
 * every forward and backward call.
 */
int sa_sketch_get_device_status(const void* workspace, void* stream);

/*
 * Measurement hook. When both handles are non-null, every later sa_sketch_forward
 * call made by this host thread records `start_event` on its stream just before the
 * main forward kernel (the tcgen05 kernel for bf16, the SIMT kernels for fp32) and
 * `stop_event` just after it; the cross-attention calls likewise around their main
 * kernel (the flash kernel for sa_stca_forward and sa_stca_keys_forward, the tcgen05
 * backward kernel for sa_stca_backward and sa_stca_keys_backward). The caller then reads that kernel's own duration with
 * cudaEventElapsedTime. Both handles are cudaEvent_t passed as void*; the caller owns
 * them. Passing two nulls turns the hook off. Returns SA_OK, or SA_ERR_INVALID_ARG if
 * exactly one handle is null.
 */
int sa_sketch_profile_events(void* start_event, void* stop_event);

/*
 * Test hook for the tensor-core GEMM that the backward is built from (bf16 operands,
 * fp32 accumulate, 128 x 128 tiles):  out[s][m][n] = sum over the K range of split s of
 * A[m][k] B[n][k], for s < splits (the caller sums the split partials).
 *   A: a_mn = 0: stored [M][K] (K contiguous); a_mn = 1: stored [K][M].
 *   B: b_mn = 0: stored [N][K];                b_mn = 1: stored [K][N].
 *   out: fp32 [splits][M][N], device. workspace: at least 256 bytes, 256-aligned, device
 *   (only its status word is used). M, N, K >= 1; the contiguous dimension of A and B a
 *   multiple of 8; N a multiple of 4; 1 <= splits <= ceil(K / 64).
 * Returns SA_OK, SA_ERR_INVALID_ARG or SA_ERR_CUDA; device errors are latched in the
 * workspace status word as for the forward.
 */
int sa_sketch_debug_gemm(const void* A, int a_mn, const void* B, int b_mn, int M, int N, int K,
                         int splits, float* out, void* workspace, void* stream);

/*
 * Candidate-to-sketch cross attention: the sketch branch of STCA, with every candidate
 * of a user reading that user's one sketch ("100,000 videos in your pocket" blog,
 * sections "2. STCA reasons at two time scales" and "3. The system makes it cheap
 * enough to matter", multi-request user-level batching). For user u and each candidate
 * c in [cand_offsets[u], cand_offsets[u+1]):
 *   q = Q_c Wq,  K_j = S_uj WK,  V_j = S_uj WV            (j < k, the sketch rows)
 *   out_c = sum_j softmax_j(q . K_j / sqrt(d)) V_j,  lse_c = log sum_j exp(q . K_j / sqrt(d))
 *
 *   Q            [n_cand, d]  bf16, device   candidates, users' groups concatenated
 *   cand_offsets [R + 1]      int64, device  0 = c_0 <= c_1 <= ... <= c_R = n_cand
 *   S            [R, k, d]    fp32, device   the users' sketches (sa_sketch_forward output)
 *   Wq, WK, WV   [d, d]       bf16, device   row-major, x W for a row vector x
 *   out          [n_cand, d]  fp32, device   output (overwritten)
 *   lse          [n_cand]     fp32, device   output, nullable
 * d in {64, 128}; 1 <= k <= SA_MAX_K; n_cand <= INT32_MAX; pointers 16-byte aligned.
 * A user without candidates reads nothing. R k_pad <= INT32_MAX (k_pad = k rounded up to
 * a multiple of 128). Both directions run sa_stca_keys_forward's and
 * sa_stca_keys_backward's kernels with the bf16 sketch as the key rows. Precision:
 * Q Wq WK^T / sqrt(d) is formed in fp32 and enters the tensor cores as a bf16 pair
 * hi + lo; the sketch and the attention weights (and in the backward their gradients)
 * enter as bf16; accumulation is fp32.
 * The workspace (sa_stca_workspace_size bytes, 256-aligned, caller-owned) holds the bf16
 * sketch (2 k_pad d bytes per user), per candidate Q Wq WK^T and the unprojected output,
 * and for the backward the gradient over the padded sketch rows; errors follow
 * sa_sketch_forward's conventions, and the device status word in the workspace is read
 * with sa_sketch_get_device_status. Enqueues on `stream`, never synchronises.
 */
size_t sa_stca_workspace_size(int R, int64_t n_cand, int k, int d, int backward);
int sa_stca_forward(const void* Q, const int64_t* cand_offsets, int R, int64_t n_cand, int d,
                    const float* S, int k, const void* Wq, const void* WK, const void* WV,
                    float* out, float* lse, void* workspace, size_t ws_bytes, void* stream);

/*
 * Gradients of the cross attention above, given dout = dL/dout [n_cand, d] (fp32,
 * device):
 *   dQ  [n_cand, d]  fp32, device   dL/dQ
 *   dS  [R, k, d]    fp32, device   dL/dS, the gradient that flows into each user's
 *                                   sketch (Sketch Attention's dsketch); zero for users
 *                                   without candidates
 *   dWq, dWK, dWV [d, d] fp32, device, summed over users
 * All outputs are overwritten. cand_offsets_host is a HOST copy of cand_offsets; it is
 * checked on the host before anything is launched (SA_ERR_BAD_OFFSETS). The forward is
 * recomputed inside. Workspace: sa_stca_workspace_size(..., backward = 1) bytes. Other arguments,
 * precision and conventions as for sa_stca_forward.
 */
int sa_stca_backward(const void* Q, const int64_t* cand_offsets, const int64_t* cand_offsets_host,
                     int R, int64_t n_cand, int d, const float* S, int k, const void* Wq,
                     const void* WK, const void* WV, const float* dout, float* dQ, float* dS,
                     float* dWq, float* dWK, float* dWV, void* workspace, size_t ws_bytes,
                     void* stream);

/*
 * Cross attention from each user's candidates to a ragged range of that user's key rows:
 * the recent branch of STCA, whose keys are the user's last 10K raw history tokens ("100,000
 * videos in your pocket" blog, section "2. STCA reasons at two time scales", recent branch).
 * For user u and each candidate c in [cand_offsets[u], cand_offsets[u+1]):
 *   q = Q_c Wq,  K_j = Kx_j WK,  V_j = Kx_j WV      (j in [key_begin[u], key_end[u]))
 *   out_c = sum_j softmax_j(q . K_j / sqrt(d)) V_j,  lse_c = log sum_j exp(q . K_j / sqrt(d))
 * A user whose range is empty gets out = 0 and lse = -inf.
 *
 *   Q            [n_cand, d]  bf16, device   candidates, users' groups concatenated
 *   cand_offsets [R + 1]      int64, device  0 = c_0 <= c_1 <= ... <= c_R = n_cand
 *   Kx           [n_keys, d]  bf16, device   key rows; for the recent branch the history X
 *                                            itself (sa_sketch_forward's input), read in place
 *   key_begin, key_end [R]    int64, device  user u's rows are Kx[key_begin[u] : key_end[u]];
 *                                            0 <= key_begin[u] <= key_end[u] <= n_keys, else
 *                                            SA_ERR_BAD_OFFSETS in the device status word.
 *                                            Ranges of different users may overlap.
 *   Wq, WK, WV   [d, d]       bf16, device   row-major, x W for a row vector x
 *   out          [n_cand, d]  fp32, device   output (overwritten)
 *   lse          [n_cand]     fp32, device   output, nullable
 * d in {64, 128}; n_cand, n_keys <= INT32_MAX; R <= SA_MAX_USERS; Q, Kx, weights and outputs
 * 16-byte aligned, key_begin / key_end 8-byte aligned. Precision: Q Wq WK^T / sqrt(d) is
 * formed in fp32 and enters the tensor cores as a bf16 pair hi + lo (about 16 significant
 * bits); the key rows and the attention weights enter as bf16; accumulation is fp32 and the
 * softmax runs in fp32 along each candidate's row with a running maximum (a flash-style
 * kernel: the scores of a candidate never leave the chip).
 * The workspace (sa_stca_keys_workspace_size bytes, 256-aligned, caller-owned) holds the
 * schedule, Q Wq WK^T and the unprojected output (about 16 d bytes per candidate); errors
 * follow sa_sketch_forward's conventions, and the device status word in the workspace is
 * read with sa_sketch_get_device_status. Enqueues on `stream`, never synchronises.
 */
size_t sa_stca_keys_workspace_size(int R, int64_t n_cand, int d, int backward);
int sa_stca_keys_forward(const void* Q, const int64_t* cand_offsets, int R, int64_t n_cand, int d,
                         const void* Kx, int64_t n_keys, const int64_t* key_begin,
                         const int64_t* key_end, const void* Wq, const void* WK, const void* WV,
                         float* out, float* lse, void* workspace, size_t ws_bytes, void* stream);

/*
 * Gradients of sa_stca_keys_forward given dout = dL/dout [n_cand, d] (fp32, device):
 *   dQ  [n_cand, d]  fp32, device   dL/dQ
 *   dKx [n_keys, d]  fp32, device   dL/dKx: for the recent branch the gradient that flows
 *                                   into the history rows; 0 on rows no range covers, a
 *                                   sum over users on rows several ranges cover
 *   dWq, dWK, dWV [d, d] fp32, device, summed over users
 * All outputs are overwritten, except dKx when accumulate is non-zero: then the
 * gradient is added into the caller's dKx (for the recent branch, straight into the
 * history gradient that sa_sketch_backward wrote, without zeroing n_keys x d floats
 * first). The forward is recomputed inside. Workspace:
 * sa_stca_keys_workspace_size(..., backward = 1) bytes. Other arguments, precision and
 * conventions as for sa_stca_keys_forward.
 */
int sa_stca_keys_backward(const void* Q, const int64_t* cand_offsets, int R, int64_t n_cand,
                          int d, const void* Kx, int64_t n_keys, const int64_t* key_begin,
                          const int64_t* key_end, const void* Wq, const void* WK, const void* WV,
                          const float* dout, float* dQ, float* dKx, int accumulate, float* dWq,
                          float* dWK, float* dWV, void* workspace, size_t ws_bytes, void* stream);

/*
 * The recent branch's key ranges over a history X laid out as for sa_sketch_forward: user
 * u's last min(n_u, L) tokens, key_begin[u] = max(offsets[u], offsets[u+1] - L) and
 * key_end[u] = offsets[u+1] ("100,000 videos in your pocket" blog, section "2. STCA
 * reasons at two time scales": the recent 10K, L = 10000). offsets [R + 1] int64, device;
 * key_begin, key_end [R] int64, device (written). L >= 0. Enqueues one kernel on `stream`;
 * offsets are not validated here (sa_stca_keys_forward checks the ranges it receives).
 * Returns SA_OK, SA_ERR_INVALID_ARG, SA_ERR_NO_DEVICE or SA_ERR_CUDA.
 */
int sa_stca_recent_ranges(const int64_t* offsets, int R, int64_t L, int64_t* key_begin,
                          int64_t* key_end, void* stream);

/*
 * Sketch cache codec. The sketch is user-only and reused across candidates and
 * requests ("100,000 videos in your pocket" blog, section "3. The system makes it cheap
 * enough to matter", low-rank caching), so it is kept packed between requests:
 *   SA_CODEC_BF16: codes [rows, d] bf16, each value rounded to nearest (ties to even);
 *   SA_CODEC_FP8:  codes [rows, d] FP8 E4M3 (finite-only, saturating at 448) of
 *                  x / s_row, with s_row = max |row| / 448 (1 for an all-zero row) in
 *                  scales [rows] fp32; scale and quotient in fp32 IEEE arithmetic;
 *                  zeros are stored as +0. Unpack: code * s_row, rounded to fp32.
 *   sketch [rows, d] fp32, device (rows = R k for R users' sketches); d in {64, 128};
 *   pointers 16-byte aligned; scales may be null for SA_CODEC_BF16.
 * Allocates nothing, enqueues one kernel on `stream`, never synchronises. Returns SA_OK,
 * SA_ERR_INVALID_ARG, SA_ERR_UNSUPPORTED or SA_ERR_CUDA.
 */
#define SA_CODEC_BF16 0
#define SA_CODEC_FP8 1
int sa_sketch_pack(const float* sketch, int64_t rows, int d, int format, void* codes,
                   float* scales, void* stream);
int sa_sketch_unpack(const void* codes, const float* scales, int64_t rows, int d, int format,
                     float* sketch, void* stream);

/* Static, human-readable name of a status code. */
const char* sa_status_string(int status);

/*
 * Test hook for the failure-detection path. It launches one block that waits on
 * an mbarrier that nothing ever arrives on. The wait uses the same bounded-wait
 * routine as the production kernels, with a limit of `budget_cycles` SM clocks.
 * When the limit runs out the kernel latches SA_ERR_TIMEOUT in `workspace`
 * (which needs >= 256 bytes) and returns. It never hangs and never traps.
 * Read the result with sa_sketch_get_device_status().
 */
int sa_sketch_debug_wait_timeout(void* workspace, long long budget_cycles, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SA_SKETCH_H */
