/*
 * bsa.h -- C ABI of the B200 (sm_100a) block-sparse attention library
 *          (libbsa_b200.so): content-aware block masks (ASA), fixed block
 *          patterns, and attention over the kept blocks.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tensors Q, K, V, O are bf16, shape [B, H, N, d], contiguous, row-major
 *    (d fastest).  LSE is fp32 [B, H, N].  Token order inside N is whatever the
 *    caller uses (the video layers are frame-major (t, y, x), x fastest).
 *  - Blocks: nb = ceil(N / blk) query blocks and nb key/value blocks (self
 *    attention).  Block i holds tokens [i*blk, min((i+1)*blk, N)); the last one
 *    may be partial.
 *  - A block mask is CSR over rows r = (b*H + h)*nb + i:
 *      row_ptr int32 [B*H*nb + 1], row_ptr[0] = 0, non-decreasing;
 *      col_idx int32 [row_ptr[B*H*nb]], each row's kv-block ids strictly
 *      ascending, each in [0, nb).
 *  - Every pointer argument is a DEVICE pointer owned by the caller unless its
 *    name ends in _host.  The library allocates no device memory: scratch comes
 *    from a caller-supplied workspace sized by the matching *_workspace_size().
 *    Workspaces must be 256-byte aligned; Q/K/V/O must be 16-byte aligned.
 *  - Every call is asynchronous on `stream` (0 = legacy default stream) unless
 *    stated otherwise, and returns a status code.  Arguments are validated on
 *    the host first: an invalid call returns an error and launches nothing.
 *    Errors found on the device (capacity overflow, malformed CSR, a bounded
 *    wait that gave up) are recorded in a per-device status word read by
 *    bsa_check_device_status().  No C++ exception crosses this interface.
 *  - Supported: d in {64, 128}; blk in {16, 32, 64, 128}; N >= 1; B, H >= 1;
 *    B*H*nb*nb < 2^31 (the backward also nb <= 4096).  The device must be
 *    sm_100 (B200).
 *
 * Typical call sequence for one attention layer (device buffers owned by the
 * caller, all calls on one stream):
 *   ws  = asa_build_mask_workspace_size(B, H, N, d, blk)     -> allocate ws
 *   cap = asa_build_mask_max_nnz(B, H, N, blk, mode, ...)    -> col_idx [cap]
 *   asa_build_mask(q, k, ..., row_ptr, col_idx, cap, ws, ws_bytes, s);
 *   bsa_forward(q, k, v, ..., row_ptr, col_idx, scale, o, lse, fws, fws_bytes, s);
 *   (training) bsa_backward(q, k, v, o, dout, lse, ..., dq, dk, dv, bws, bws_bytes, s);
 *   bsa_check_device_status(s)   -- once per step or when debugging
 * pattern_mask replaces asa_build_mask for the fixed patterns.
 *
 * Sources (web pages on the method):
 *  [BLADE]   "BLADE: Block-Sparse Attention Meets Step Distillation for
 *            Efficient Video Generation" (digest: abstract; 技术框架;
 *            方法详解 / 关键设计)
 *  [SvDiT]   "Sparse-vDiT: Sparse Attention Acceleration for Video Diffusion
 *            Transformers" (blog: 核心公式; 四种注意力模式 table; 模型组件)
 *  [EvDiT]   "Efficient-vDiT: Efficient Video Diffusion Transformers With
 *            Attention Tile" (blog: 3.1 注意力图块化)
 */
#ifndef BSA_B200_H
#define BSA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* bsa_stream_t; /* same object as cudaStream_t */

/* ---- status codes ------------------------------------------------------- */
#define BSA_OK               0
#define BSA_ERR_INVALID_ARG (-1) /* null pointer, non-positive size, bad mode   */
#define BSA_ERR_UNSUPPORTED (-2) /* d, blk, alignment or size outside support   */
#define BSA_ERR_CAPACITY    (-3) /* col_idx capacity too small for the mask     */
#define BSA_ERR_CUDA        (-4) /* a CUDA runtime call or launch failed        */
#define BSA_ERR_TIMEOUT     (-5) /* a device-side bounded wait gave up          */
#define BSA_ERR_CSR         (-6) /* device saw a block index outside [0, nb)    */
#define BSA_ERR_WORKSPACE   (-7) /* workspace null, too small or misaligned     */

#define BSA_MODE_TOPK 0
#define BSA_MODE_MASS 1

#define BSA_PATTERN_FULL      0 /* M0  [SvDiT] every block                          */
#define BSA_PATTERN_SKIP      1 /* M1  [SvDiT] head skipped, output zero            */
#define BSA_PATTERN_DIAG      2 /* M2  [SvDiT] diagonal band (intra-frame)          */
#define BSA_PATTERN_MULTIDIAG 3 /* M3  [SvDiT] diagonals at frame offsets           */
#define BSA_PATTERN_STRIPE    4 /* M4  [SvDiT] vertical stripes (global tokens)     */
#define BSA_PATTERN_TILE3D    5 /*     [EvDiT] frame tiles + global frames          */

/* ---- ASA: content-aware block mask --------------------------------------
 * [BLADE] ASA generates, per input, a sparsity mask that keeps the block pairs
 * whose mutual relevance is high.  The pages do not define the score; this
 * library computes, per (b, h):
 *   1. pooled q̄_i, k̄_j = mean of the block's valid rows (fp32 accumulation);
 *   2. s_ij = q̄_i·k̄_j·scale (scale = 1/sqrt(d) when softmax_scale <= 0, the
 *      attention scale of [SvDiT] 核心公式); p_i = softmax_j s_i over all nb;
 *   3. order j by (p desc, j asc);
 *      mode BSA_MODE_TOPK: the first `topk`;
 *      mode BSA_MODE_MASS: the shortest prefix with cumulative p >= mass_tau;
 *   4. cap: when max_keep_ratio > 0 keep at most max(1, floor(max_keep_ratio*nb));
 *   5. union with the diagonal block i (keep_diag != 0) and blocks
 *      [0, n_sink_blocks);
 *   6. write CSR (row_ptr, col_idx ascending).
 * Two kernels: pooling (reads q and k once), then scores, selection and the
 * CSR write together (the row offsets by a decoupled look-back across CTAs).
 * Selection runs in fp32 on the device: rows whose result depends on scores
 * within fp32 rounding of the cut may differ from an exact evaluation.
 * q, k: bf16 [B,H,N,d].  col_capacity: entries available in col_idx; if the mask
 * needs more, entries past the capacity are not written and the device status
 * becomes BSA_ERR_CAPACITY.  asa_build_mask_max_nnz() gives a bound that never
 * overflows.  Workspace: asa_build_mask_workspace_size() bytes. */
size_t  asa_build_mask_workspace_size(int B, int H, int N, int d, int blk);
int64_t asa_build_mask_max_nnz(int B, int H, int N, int blk, int mode, int topk,
                               float max_keep_ratio, int keep_diag, int n_sink_blocks);
int asa_build_mask(const void* q, const void* k, int B, int H, int N, int d, int blk,
                   int mode, int topk, float mass_tau, float max_keep_ratio,
                   int keep_diag, int n_sink_blocks, float softmax_scale,
                   int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity,
                   void* workspace, size_t ws_bytes, bsa_stream_t stream);

/* ---- ASA mask without device allocation ---------------------------------
 * No counterpart on the pages: an interface addition for callers that may not
 * call cudaMalloc -- e.g. code embedded in a host framework or inference engine
 * that owns all device memory and forbids allocation while it runs, or a
 * real-time path where an allocation's implicit synchronization is not
 * acceptable.  Same arguments and results as asa_build_mask, without the
 * workspace: the scratch is a fixed array of BSA_ASA_NOALLOC_MAX_WORKSPACE
 * bytes that the library keeps in the memory of every GPU that loads it, until
 * the process exits.  Shapes whose asa_build_mask_workspace_size() exceeds it
 * are rejected with BSA_ERR_WORKSPACE and nothing is launched (16 MiB covers,
 * e.g., B1 H12 N32760 d128 and B2 H48 N17776 d64 at blk 64).  This function
 * calls no cudaMalloc, cudaFree or other allocating routine.
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call before
 * any stream capture begins.  The address is kept for the life of the
 * process: do not reset the device (cudaDeviceReset) between calls.  Every
 * call on a device shares the one array, and the array keeps the last call's
 * contents (each call clears, on the device, the part that must start at
 * zero): calls that may overlap on the GPU -- on different streams, or from
 * different host threads without ordering -- race on it and must be
 * serialized by the caller. */
#define BSA_ASA_NOALLOC_MAX_WORKSPACE (16u << 20)
int asa_build_mask_noalloc(const void* q, const void* k, int B, int H, int N, int d, int blk,
                           int mode, int topk, float mass_tau, float max_keep_ratio,
                           int keep_diag, int n_sink_blocks, float softmax_scale,
                           int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity,
                           bsa_stream_t stream);

/* ---- fixed patterns ------------------------------------------------------
 * [SvDiT] 四种注意力模式 (M0 full, M1 skip, M2 diagonal, M3 multi-diagonal,
 * M4 vertical stripe) and [EvDiT] 3.1 (3D attention tile), one pattern per
 * head, rows replicated over b.  Block (i, j) is kept when some token pair
 * (t in block i, u in block j, both < N) satisfies the pattern's rule, with
 * S = frame_tokens:
 *   FULL      always;            SKIP  never (row empty -> O = 0, LSE = -inf);
 *   DIAG      |i - j| <= band_w  (block bandwidth);
 *   MULTIDIAG |u - t - f*S| <= band_w*blk for some f in [f_lo, f_hi];
 *   STRIPE    (u mod S) < stripe_blocks*blk   (leading tokens of every frame);
 *   TILE3D    floor(u/S) == floor(t/S) or floor(u/S) < tile_global_frames.
 * head_pattern_host: HOST int32 [H].  If nnz_out_host is non-NULL the call
 * synchronizes `stream` once after counting, stores the mask's nnz there, and
 * returns BSA_ERR_CAPACITY (writing no col_idx) when col_capacity < nnz.  With
 * nnz_out_host NULL the call is fully asynchronous and an overflow is reported
 * through the device status.  No workspace.  band_w*blk above 2^24 or
 * frame_tokens above 2^28 gives BSA_ERR_UNSUPPORTED. */
int pattern_mask(const int32_t* head_pattern_host, int B, int H, int N, int blk,
                 int band_w, int frame_tokens, int f_lo, int f_hi, int stripe_blocks,
                 int tile_global_frames, int32_t* row_ptr, int32_t* col_idx,
                 int64_t col_capacity, int64_t* nnz_out_host, bsa_stream_t stream);

/* ---- attention over kept blocks -------------------------------------------
 * [SvDiT] 核心公式: O = softmax(Q Kᵀ · scale) V per head, here for each query
 * token t of block i over the key tokens (< N) of the blocks listed in CSR row
 * (b*H + h)*nb + i only ([BLADE] abstract: computation focused on the kept
 * blocks).  scale = 1/sqrt(d) when softmax_scale <= 0.
 * Output: o bf16 [B,H,N,d] (round to nearest even), lse fp32 [B,H,N] =
 * ln Σ_u exp(q_t·k_u·scale); an empty row gives o = 0 and lse = -inf
 * ([SvDiT] M1: a skipped head outputs zero).  lse may be NULL.
 * Accumulation is fp32 on the tensor cores (tcgen05, operands from TMA-loaded
 * shared memory).  A CSR block id outside [0, nb) is skipped and flagged
 * (BSA_ERR_CSR in the device status).  Workspace: bsa_forward_workspace_size()
 * bytes (256, 4-byte aligned) holding a counter from which the persistent
 * CTAs take work items, so that faster SMs take more; it is zeroed on `stream`
 * before the launch, and concurrent calls need separate workspaces.  NULL is
 * accepted: items are then dealt round-robin.  A non-NULL workspace under 4
 * bytes or misaligned gives BSA_ERR_WORKSPACE. */
size_t bsa_forward_workspace_size(int B, int H, int N, int d, int blk);
int bsa_forward(const void* q, const void* k, const void* v, int B, int H, int N, int d,
                int blk, const int32_t* row_ptr, const int32_t* col_idx,
                float softmax_scale, void* o, float* lse,
                void* workspace, size_t ws_bytes, bsa_stream_t stream);

/* bsa_forward that also writes, when o_residual is not NULL (bf16
 * [B,H,N,d], 16-byte aligned, caller-owned), each element's fp32 result minus
 * its bf16 rounding in o, rounded to bf16: o + o_residual carries the fp32 O
 * to about 2^-16 relative.  bsa_backward_residual takes it to form D = dO.O
 * from the fp32 O (an empty row gives o_residual = 0).  The pages have no
 * counterpart; it is the training path's precision option (see
 * bsa_backward_residual).  Misaligned o_residual: BSA_ERR_UNSUPPORTED. */
int bsa_forward_residual(const void* q, const void* k, const void* v, int B, int H, int N, int d,
                         int blk, const int32_t* row_ptr, const int32_t* col_idx,
                         float softmax_scale, void* o, float* lse, void* o_residual,
                         void* workspace, size_t ws_bytes, bsa_stream_t stream);

/* ---- gradients of attention over kept blocks --------------------------------
 * [BLADE] 技术框架: ASA is trained jointly with the step distillation, so the
 * attention over the kept blocks is differentiated.  For a given dO (bf16
 * [B,H,N,d]) this returns the gradient of the bsa_forward definition with
 * respect to q, k and v, with the block mask held constant (its selection
 * carries no gradient) and no gradient into lse:
 *     P_tu = exp(scale q_t.k_u - lse_t)  over the listed key tokens u < N,
 *     D_t = dO_t . O_t,   dS_tu = P_tu (dO_t . v_u - D_t),
 *     dq_t = scale sum_u dS_tu k_u,  dk_u = scale sum_t dS_tu q_t,
 *     dv_u = sum_t P_tu dO_t.
 * o and lse are the outputs of bsa_forward on the same q, k, v, mask and
 * scale (lse must not be NULL).  Each CSR row must be strictly ascending,
 * nb must be at most 4096 and B*H*N*d/8 below 2^31.  A token whose row lists nothing gets dq = 0 and
 * adds nothing; a key token no row reaches gets dk = dv = 0.  Outputs dq, dk,
 * dv are bf16 [B,H,N,d] (round to nearest even), each written once (no
 * atomics: the result does not depend on scheduling); accumulation is fp32 on
 * the tensor cores.  Workspace: bsa_backward_workspace_size() bytes, 256-byte
 * aligned, holding D (fp32 [B,H,N]).  Asynchronous on `stream`.  A CSR block
 * id outside [0, nb) is skipped and flagged (BSA_ERR_CSR in the device
 * status). */
size_t bsa_backward_workspace_size(int B, int H, int N, int d, int blk);
int bsa_backward(const void* q, const void* k, const void* v, const void* o, const void* dout,
                 const float* lse, int B, int H, int N, int d, int blk,
                 const int32_t* row_ptr, const int32_t* col_idx, float softmax_scale,
                 void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes,
                 bsa_stream_t stream);

/* bsa_backward with the forward's rounding residual (bsa_forward_residual;
 * NULL: the same as bsa_backward).  With it D_t = dO_t.(o_t + o_residual_t)
 * comes from the fp32 O; without it D comes from the bf16 o, whose rounding
 * (up to 2^-8 relative per element) then reaches dq through D -- on peaked
 * attention, where dP - D nearly cancels, that rounding dominates dq's error.
 * dk and dv are barely affected.  Misaligned o_residual: BSA_ERR_UNSUPPORTED. */
int bsa_backward_residual(const void* q, const void* k, const void* v, const void* o,
                          const void* o_residual, const void* dout, const float* lse, int B,
                          int H, int N, int d, int blk, const int32_t* row_ptr,
                          const int32_t* col_idx, float softmax_scale, void* dq, void* dk,
                          void* dv, void* workspace, size_t ws_bytes, bsa_stream_t stream);

/* ---- Sparse-vDiT offline pattern search (diagnostic) ------------------------
 * Sparse-vDiT blog, "核心公式 / 离线搜索损失函数", "注意力模式选择" and
 * Algorithm 1: for each head and candidate pattern i,
 *     L_i = MSE(O_i - O_0) + lambda * (1 - S_i),
 * O_0 the output of full attention (M0), S_i the pattern's sparsity; the head
 * keeps full attention when L_i > eps for every candidate, else takes the
 * candidate of the smallest L_i.  Readings: MSE averages over all B*N*d
 * elements of the head; S = 1 - (computed query/key token pairs) / (B*N*N),
 * a kept block pair (i, j) counting n_q(i) * n_k(j) valid tokens; ties go to
 * the candidate listed first.  The O_i come from bsa_forward on the masks of
 * pattern_mask; the real search runs on a model's activations, which this
 * library does not hold.
 *
 * attention_head_mse: mse[h] (device, [H] doubles) for bf16 O_ref, O
 * [B,H,N,d] (device, 16-byte aligned), d in {64, 128}.  Deterministic
 * (fixed-order sums).  Workspace: attention_head_mse_workspace_size() bytes,
 * 256-byte aligned.  Asynchronous on `stream`.
 * csr_head_sparsity: sparsity[h] (device, [H] doubles) of a CSR block mask
 * over B*H*nb rows (device; each row's block ids ascending, as bsa_forward
 * requires); col_idx may be NULL when the mask is empty.  Workspace:
 * csr_head_sparsity_workspace_size(H) bytes, 256-byte aligned.  Asynchronous.
 * pattern_search_select: host arrays only, no device work.  mse, sparsity
 * [P][H] (candidate-major), candidates [P] pattern ids; writes choice [H]
 * (a candidate id or BSA_PATTERN_FULL) and, when loss is not NULL, L [P][H]. */
size_t attention_head_mse_workspace_size(int B, int H, int N, int d);
int attention_head_mse(const void* o_ref, const void* o, int B, int H, int N, int d, double* mse,
                       void* workspace, size_t ws_bytes, bsa_stream_t stream);
size_t csr_head_sparsity_workspace_size(int H);
int csr_head_sparsity(const int32_t* row_ptr, const int32_t* col_idx, int B, int H, int N, int blk,
                      double* sparsity, void* workspace, size_t ws_bytes, bsa_stream_t stream);
int pattern_search_select(const double* mse, const double* sparsity, const int32_t* candidates,
                          int P, int H, double lambda, double eps, double* loss, int32_t* choice);

/* ---- CSR check (host) ---------------------------------------------------------
 * bsa_validate_csr_host checks a block mask held in HOST memory against the
 * conventions above: row_ptr[0] = 0, non-decreasing, row_ptr[rows] <= col_len
 * (the length of col_idx_host), every block id in [0, nb) and each row strictly
 * ascending (as bsa_backward requires; bsa_forward tolerates any order).
 * Returns BSA_OK, or BSA_ERR_CSR with the first offending row in
 * *bad_row_host (may be NULL; -1 when the mask is valid).  No device work. */
int bsa_validate_csr_host(const int32_t* row_ptr_host, const int32_t* col_idx_host, int64_t rows,
                          int nb, int64_t col_len, int64_t* bad_row_host);

/* ---- status ----------------------------------------------------------------
 * bsa_check_device_status synchronizes `stream`, returns the first error any
 * kernel of this library recorded on the current device since the last check
 * (BSA_OK if none), and clears it.  bsa_status_string never returns NULL. */
int bsa_check_device_status(bsa_stream_t stream);
const char* bsa_status_string(int status);
/* Diagnostics: y[i] = the attention kernel's FMA-pipe exponential 2^x[i]
 * (Cody-Waite reduction + degree-3 minimax polynomial, relative error below
 * 1e-4 for x in [-125, 126]; below that the result is a non-negative value
 * under 2^-124).  Device
 * pointers, n floats; asynchronous on `stream`.  For testing the kernel's
 * arithmetic against the CUDA math library; no counterpart on the pages. */
int bsa_debug_exp2_poly(const float* x, float* y, int n, bsa_stream_t stream);
/* Diagnostics: failure detection without a GPU fault.  One thread waits, with
 * the bounded wait that every kernel of this library uses on its mbarriers,
 * on a phase that completes only when arrive_first is nonzero.  Without the
 * arrive the wait gives up after limit_ns nanoseconds (at most 10 s, else
 * BSA_ERR_INVALID_ARG), BSA_ERR_TIMEOUT is recorded in the device status and
 * the kernel returns: the context stays usable.  waited_ns (device, 8-byte
 * aligned, may be NULL) receives how long the wait took.  Asynchronous on
 * `stream`.  No counterpart on the pages. */
int bsa_debug_wait_timeout(unsigned long long limit_ns, int arrive_first,
                           unsigned long long* waited_ns, bsa_stream_t stream);
/* Library version as major*10000 + minor*100 + patch. */
int bsa_version(void);

#ifdef __cplusplus
}
#endif
#endif /* BSA_B200_H */
