/*
 * lc_bsa.h -- C ABI of liblcbsa.so: block-sparse 3D-RoPE self-attention over
 * video latent tokens (the 3D self-attention of the LongCat-Video diffusion
 * transformer), for NVIDIA B200 (sm_100a).
 *
 * What the operation is (sources are the pages the method is described on):
 *   - "longcat-video-rs" (code.brandonhubbard.com), header card and section
 *     03-01 "Partitioned 3D-RoPE (16T+24H+24W)": every 64-D head is split into
 *     16 temporal, 24 height and 24 width channels, rotated as complex pairs
 *     by the token's (t, h, w) position.
 *   - same page, section 03-03 "Block-Sparse & Multi-Audio" and the section 02
 *     table row "Block-Sparse Self-Attention (block=64, local=2, stride=4)":
 *     a query block attends a local window of key blocks plus strided global
 *     key blocks.
 *   - "美团视频生成模型来了！一出手就是开源 SOTA" (myzaker / QbitAI), section
 *     "背后技术原理": condition frames precede the noisy frames on the time
 *     axis; condition tokens are not affected by noise tokens and their K/V
 *     can be cached and reused.
 *
 * Readings where the pages are silent (same as the test oracle's):
 *   token n of the full sequence sits at t = n/(H*W), h = (n/W)%H, w = n%W;
 *   RoPE pair k of an axis of width d turns by pos*theta^(-2k/d), pairs are
 *   adjacent channels (c, c+1), axes in the order T, H, W;
 *   a block is 64 consecutive tokens of one segment (the first Nc = n_cond*H*W
 *   tokens are the condition segment, the rest the noisy segment; the last
 *   block of a segment may be short);
 *   noisy block i attends noisy block j iff |i-j| <= local or
 *   (stride > 0 and j % stride == 0); stride == 1 is dense, stride <= 0 means
 *   no global blocks;
 *   condition queries attend every condition key and no noisy key; noisy
 *   queries attend every condition key plus their noisy blocks;
 *   softmax scale 1/sqrt(head_dim) unless given.
 *
 * Conventions shared by every entry point:
 *   - Tensors are contiguous [B, N, heads, head_dim] ("BMHK"), tokens ordered
 *     t-major, then h, then w.  Device pointers, 16-byte aligned.  LSE is
 *     [B, heads, Nq] fp32, natural log.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Every call is stream ordered and returns without waiting for the GPU,
 *     except lc_bsa_plan_info, lc_bsa_plan_copy_csr / _csc, lc_rope3d_copy_tables and
 *     lc_last_device_status, which synchronise the stream.
 *   - Errors are returned as lc_status; argument errors are detected before any
 *     GPU work is queued.  No C++ exception crosses this boundary.
 *   - The caller owns q/k/v/out/lse.  The library owns the memory behind plan
 *     and rope handles (allocated stream-ordered on the given stream, released
 *     by the matching *_destroy on its stream).
 *   - There is no CPU fallback: on a machine without a usable sm_100 GPU the
 *     calls that need one return LC_ERR_CUDA.
 *   - v1 supports block = 64 and head_dim = 64 with RoPE channel split
 *     16/24/24; other values return LC_ERR_UNSUPPORTED.
 */
#ifndef LC_BSA_H
#define LC_BSA_H

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LC_OK = 0,
    LC_ERR_INVALID_ARGUMENT = 1,  /* null pointer, bad size, misaligned pointer, mismatch */
    LC_ERR_UNSUPPORTED = 2,       /* valid but not implemented (block or head_dim != 64 ...) */
    LC_ERR_CUDA = 3,              /* a CUDA runtime/driver call failed (incl. no device) */
    LC_ERR_OUT_OF_MEMORY = 4,     /* device allocation failed */
    LC_ERR_TIMEOUT = 5,           /* a bounded in-kernel wait gave up (device status) */
    LC_ERR_DEVICE_CHECK = 6       /* an in-kernel bounds/consistency check failed (device status) */
} lc_status;

typedef enum {
    LC_DTYPE_BF16 = 0,   /* tcgen05 tensor-core kernel, fp32 accumulation */
    LC_DTYPE_F32 = 1     /* fp32 SIMT kernel (exact-arithmetic reference speed path) */
} lc_dtype;

typedef struct lc_bsa_plan_s *lc_bsa_plan;   /* opaque, device resident, read-only once built */
typedef struct lc_rope3d_s *lc_rope3d;       /* opaque, device resident */

/* Summary of a plan; returned by lc_bsa_plan_info. */
typedef struct {
    int num_q_blocks;          /* Cb + Nb: rows of the block CSR */
    int num_cond_blocks;       /* Cb = ceil(Nc / block) */
    int num_noisy_blocks;      /* Nb = ceil(Nn / block) */
    long long nnz;             /* entries of the block CSR */
    int n_cond_tokens;         /* Nc = n_cond_frames * H * W */
    int n_noisy_tokens;        /* Nn = (T - n_cond_frames) * H * W */
    long long attended_token_pairs;        /* per head, all queries (lc_bsa_forward) */
    long long attended_token_pairs_noisy;  /* per head, noisy queries (lc_bsa_forward_cached) */
} lc_bsa_plan_info_t;

/*
 * lc_bsa_plan_create -- build, on the device, the block-sparse pattern of a
 * (T, H, W) latent video with n_cond_frames condition frames: for each query
 * block the sorted list of attended key blocks (block CSR, key ids 0..Cb-1 for
 * condition blocks then Cb+j for noisy block j), plus the kernel's internal
 * work lists.  Source: "longcat-video-rs" section 03-03 and the section 02
 * table row (local window + strided global blocks, block=64); myzaker / QbitAI
 * "背后技术原理" (condition frames first, isolated from noise).
 *   T: latent frames including condition frames (T > n_cond_frames >= 0: the
 *      frames to generate are never empty, so n_cond_frames == T is refused);
 *   block: 64; local >= 0; stride: <= 0 none, 1 dense, > 1 strided globals.
 * Errors: LC_ERR_INVALID_ARGUMENT (out NULL, T/H/W <= 0, local < 0,
 * n_cond_frames outside [0, T), token count >= 2^31), LC_ERR_UNSUPPORTED
 * (block != 64), LC_ERR_OUT_OF_MEMORY, LC_ERR_CUDA.  *out is set only on LC_OK.
 */
lc_status lc_bsa_plan_create(lc_bsa_plan *out, int T, int H, int W, int block, int local,
                             int stride, int n_cond_frames, void *stream);

/* Release a plan (stream ordered on `stream`).  NULL is accepted. */
lc_status lc_bsa_plan_destroy(lc_bsa_plan plan, void *stream);

/* Sizes of a plan.  Waits for the plan's construction to finish. */
lc_status lc_bsa_plan_info(lc_bsa_plan plan, lc_bsa_plan_info_t *info);

/* Copy the transpose of the block CSR (CSC) to host memory:
 * col_ptr_host[num_q_blocks + 1], row_idx_host[nnz] (int32): for key block c,
 * the ascending query blocks that attend it (the backward pass walks these).
 * Synchronises `stream`.  For checking the plan. */
lc_status lc_bsa_plan_copy_csc(lc_bsa_plan plan, int *col_ptr_host, int *row_idx_host,
                               void *stream);

/* Copy the block CSR to host memory: row_ptr_host[num_q_blocks + 1],
 * col_idx_host[nnz] (int32).  Synchronises `stream`.  For checking the plan. */
lc_status lc_bsa_plan_copy_csr(lc_bsa_plan plan, int *row_ptr_host, int *col_idx_host,
                               void *stream);

/*
 * lc_rope3d_tables -- per-axis cos/sin tables of the partitioned 3D-RoPE
 * ("longcat-video-rs" header card and section 03-01): for axis a in (T, H, W)
 * of width dim_a and pair k < dim_a/2, angle = pos * theta^(-2k/dim_a), pos in
 * [0, T), [0, H), [0, W).  Computed in fp64 on the device, stored fp32.
 * dim_t + dim_h + dim_w is the head dimension; v1 needs (16, 24, 24).
 * Errors: LC_ERR_INVALID_ARGUMENT (out NULL, sizes <= 0, odd dims, theta <= 0),
 * LC_ERR_UNSUPPORTED (dims other than 16/24/24), LC_ERR_OUT_OF_MEMORY, LC_ERR_CUDA.
 */
lc_status lc_rope3d_tables(lc_rope3d *out, int T, int H, int W, double theta,
                           int dim_t, int dim_h, int dim_w, void *stream);

/* Release rope tables (stream ordered).  NULL is accepted. */
lc_status lc_rope3d_destroy(lc_rope3d rope, void *stream);

/* Copy the tables to host memory as fp32, in this order: cos_t[T][dim_t/2],
 * sin_t[T][dim_t/2], cos_h[H][dim_h/2], sin_h[H][dim_h/2], cos_w[W][dim_w/2],
 * sin_w[W][dim_w/2].  `host` holds (T*dim_t + H*dim_h + W*dim_w) floats.
 * Synchronises `stream`. */
lc_status lc_rope3d_copy_tables(lc_rope3d rope, float *host, void *stream);

/*
 * lc_rope3d_apply -- rotate x [B, ntok, heads, head_dim] by the partitioned
 * 3D-RoPE into out (same shape and dtype; out == x is allowed).  Token n of x is
 * token n + tok_offset of the full sequence.  The standalone form of the
 * rotation that the attention entry points fuse into their Q/K tile loads
 * ("longcat-video-rs" section 02 row "3D-RoPE Spatiotemporal Frequency & Token
 * Rotation", section 03-01).  Requires tok_offset + ntok <= T*H*W of the tables.
 */
lc_status lc_rope3d_apply(const void *x, void *out, int batch, long long ntok, int heads,
                          int head_dim, long long tok_offset, lc_dtype dtype,
                          lc_rope3d rope, void *stream);

/* lc_rope3d_apply with the RMSNorm of the attention modules ahead of the
 * rotation: out = R(norm(x)), norm(x) = x / sqrt(mean(x^2) + norm_eps) * w
 * per token and head (norm_weight: device fp32 [head_dim], or NULL for the
 * plain rotation).  The same arithmetic as every rotation inside the
 * attention entry points, so a tensor prepared here gives those calls the
 * same bits (LC_FLAG_Q_ROTATED / LC_FLAG_K_ROTATED). */
lc_status lc_rope3d_apply_ex(const void *x, void *out, int batch, long long ntok, int heads,
                             int head_dim, long long tok_offset, lc_dtype dtype,
                             const float *norm_weight, float norm_eps, lc_rope3d rope,
                             void *stream);

/*
 * lc_bsa_forward -- out = softmax(mask(scale * R(q) R(k)^T)) v over the whole
 * sequence of N = T*H*W tokens, with R the 3D-RoPE of `rope` and the mask of
 * `plan`; optionally lse (nullable).  q, k, v, out: [batch, N, heads, head_dim]
 * of `dtype`; lse: [batch, heads, N] fp32.  softmax_scale <= 0 means
 * 1/sqrt(head_dim).  plan and rope must describe the same (T, H, W).
 * Errors: LC_ERR_INVALID_ARGUMENT (NULL tensors or handles, batch/heads <= 0,
 * pointers not 16-byte aligned, plan/rope grid mismatch), LC_ERR_UNSUPPORTED
 * (head_dim != 64), LC_ERR_CUDA (launch failure).  In-kernel faults of the
 * bounded waits or checks are reported by lc_last_device_status.
 */
lc_status lc_bsa_forward(const void *q, const void *k, const void *v, void *out, float *lse,
                         int batch, int heads, int head_dim, lc_dtype dtype,
                         float softmax_scale, lc_bsa_plan plan, lc_rope3d rope, void *stream);

/*
 * lc_bsa_forward_cached -- the same attention for the noisy queries only, with
 * the condition tokens' K/V supplied separately (the KV-cache form of myzaker /
 * QbitAI "背后技术原理").  q, k, v, out: [batch, Nn, heads, head_dim] (noisy
 * tokens); cond_k, cond_v: [batch, Nc, heads, head_dim], pre-RoPE like k (they
 * are rotated with t in [0, n_cond_frames)); lse: [batch, heads, Nn] or NULL.
 * With n_cond_frames == 0, cond_k/cond_v may be NULL.  Errors as lc_bsa_forward.
 */
lc_status lc_bsa_forward_cached(const void *q, const void *k, const void *v,
                                const void *cond_k, const void *cond_v, void *out,
                                float *lse, int batch, int heads, int head_dim,
                                lc_dtype dtype, float softmax_scale, lc_bsa_plan plan,
                                lc_rope3d rope, void *stream);

/* Flags of lc_bsa_opts. */
#define LC_FLAG_COND_K_ROTATED 1u  /* cond_k already holds R(k) (lc_bsa_cond_cache) */
#define LC_FLAG_Q_ROTATED 2u       /* q already holds R(norm_q(q)) (lc_bsa_forward_shard) */
#define LC_FLAG_K_ROTATED 4u       /* k already holds R(norm_k(k)) (lc_bsa_forward_shard) */
#define LC_FLAG_KEEP_EMPTY_ROWS 8u /* lc_bsa_forward_shard: rows of work groups without keys
                                      in the shard are left as they are (not set to 0, -inf) */
#define LC_FLAG_OVERLAP_PREVIOUS 16u /* lc_bsa_forward_shard: the launch may start while the
                                        previous kernel on the stream is still finishing */

/*
 * Options of the _ex entry points and of lc_bsa_cond_cache.  A NULL options
 * pointer, or a zero-initialised struct, means none.
 *   flags:          LC_FLAG_COND_K_ROTATED (lc_bsa_forward_cached_ex only).
 *   q_norm_weight,  device fp32 [head_dim]: RMSNorm of q (resp. k and cond_k)
 *   k_norm_weight:  ahead of the 3D-RoPE, x / sqrt(mean(x^2) + norm_eps) * w
 *                   per token and head over the head's channels (myzaker /
 *                   QbitAI "背后技术原理": RMSNorm in the attention modules).
 *                   NULL: no norm.  4-byte aligned.
 *   norm_eps:       >= 0 and finite; used only with a weight.
 * The norm is fused into the same per-row rotation every entry point applies
 * (in the tile loads, the one-pass K rotation and the fp32 kernel).
 */
typedef struct {
    unsigned flags;
    const float *q_norm_weight;
    const float *k_norm_weight;
    float norm_eps;
} lc_bsa_opts;

/* lc_bsa_forward with options (RMSNorm of q and k).  Flags must be 0.
 * Errors as lc_bsa_forward, plus LC_ERR_INVALID_ARGUMENT for bad options. */
lc_status lc_bsa_forward_ex(const void *q, const void *k, const void *v, void *out, float *lse,
                            int batch, int heads, int head_dim, lc_dtype dtype,
                            float softmax_scale, const lc_bsa_opts *opts, lc_bsa_plan plan,
                            lc_rope3d rope, void *stream);

/*
 * lc_bsa_forward_cached_ex -- lc_bsa_forward_cached with options.  With
 * LC_FLAG_COND_K_ROTATED, cond_k is taken as already normalised and rotated
 * (the cond_k_rot output of lc_bsa_cond_cache with the same k_norm_weight) and
 * is used as is, so a cache built once serves every later call; the results
 * equal those of the same call on the raw cond_k bit for bit.  Unknown flag
 * bits or bad options: LC_ERR_INVALID_ARGUMENT; other errors as
 * lc_bsa_forward.
 */
lc_status lc_bsa_forward_cached_ex(const void *q, const void *k, const void *v,
                                   const void *cond_k, const void *cond_v, void *out,
                                   float *lse, int batch, int heads, int head_dim,
                                   lc_dtype dtype, float softmax_scale, const lc_bsa_opts *opts,
                                   lc_bsa_plan plan, lc_rope3d rope, void *stream);

/*
 * lc_bsa_cond_cache -- the producer side of the condition-token KV cache
 * (myzaker / QbitAI "背后技术原理", on the block attention with a KV cache:
 * condition tokens never attend noise tokens, so their K/V features, and
 * their own attention outputs, are computed once and reused at every later
 * denoising step).  From the condition tokens' pre-RoPE cond_k it writes
 * cond_k_rot = R(cond_k) with t in [0, n_cond_frames), the exact values the
 * attention entry points rotate internally, for lc_bsa_forward_cached_ex with
 * LC_FLAG_COND_K_ROTATED.  If cond_out is not NULL it also computes the
 * condition tokens' attention (condition queries over condition keys, the
 * condition rows of lc_bsa_forward on the whole sequence) into cond_out and,
 * if cond_lse is not NULL, their lse.  opts (nullable, flags 0) carries the
 * RMSNorm weights: cond_k_rot then holds R(norm_k(cond_k)) and cond_q is
 * normalised with q_norm_weight, as in lc_bsa_forward_ex.
 *   cond_q, cond_k, cond_v, cond_k_rot, cond_out: [batch, Nc, heads, head_dim]
 *   of dtype, 16-byte aligned; cond_lse: [batch, heads, Nc] fp32.  cond_q and
 *   cond_v are read only when cond_out is given (else they may be NULL).
 *   cond_k_rot must not overlap cond_k; the caller owns every buffer.
 * With n_cond_frames == 0 there is nothing to do (LC_OK).  Errors as
 * lc_bsa_forward.
 */
lc_status lc_bsa_cond_cache(const void *cond_q, const void *cond_k, const void *cond_v,
                            void *cond_k_rot, void *cond_out, float *cond_lse, int batch,
                            int heads, int head_dim, lc_dtype dtype, float softmax_scale,
                            const lc_bsa_opts *opts, lc_bsa_plan plan, lc_rope3d rope,
                            void *stream);

/*
 * lc_bsa_backward -- gradients of lc_bsa_forward (whole sequence) for the
 * training path: the SimpleTuner page ("Guia de Início Rápido do LongCat-Video
 * Edit", section "2) Mudanças no config") fine-tunes the model with LoRA and
 * gradient checkpointing.  Given the forward's inputs q, k, v, its output
 * `out` and lse (natural log, [batch, heads, N] fp32, as lc_bsa_forward wrote
 * them) and the output gradient dout, writes
 *   dv = P^T dout,  dS = P * (dout v^T - rowsum(dout * out)),
 *   dq = norm_q^T(R^T(scale dS k')),  dk = norm_k^T(R^T(scale dS^T q'))
 * over the attended pairs of `plan`, with P = exp(scale q' k'^T - lse) and
 * q' = R(norm_q(q)), k' = R(norm_k(k)) as in the forward (opts: the same
 * RMSNorm weights as the forward, flags 0; weight gradients are not
 * produced).  All tensors [batch, N, heads, head_dim] of dtype, 16-byte
 * aligned, caller owned; dq / dk / dv must not overlap the inputs.  fp32
 * arithmetic for both dtypes (bf16 tensors are converted on load and the
 * gradients rounded on store).  Scratch: batch * heads * N floats from the
 * library's pool.  Errors as lc_bsa_forward; batch or heads above 65535:
 * LC_ERR_UNSUPPORTED.
 */
lc_status lc_bsa_backward(const void *q, const void *k, const void *v, const void *out,
                          const float *lse, const void *dout, void *dq, void *dk, void *dv,
                          int batch, int heads, int head_dim, lc_dtype dtype,
                          float softmax_scale, const lc_bsa_opts *opts, lc_bsa_plan plan,
                          lc_rope3d rope, void *stream);

/*
 * lc_bsa_forward_noalloc -- lc_bsa_forward for callers that cannot allocate
 * device memory during the call: an application whose allocator owns all of
 * the GPU's memory up front, a serving loop that forbids allocations after
 * warm-up, or code that must not add memory operations to a stream.  (The
 * pages describe no such entry point; it is an addition of this library.)
 * Same arguments, layouts, results and errors as lc_bsa_forward.  It allocates
 * nothing: the tensor-core kernel's scheduler counter and status word live in
 * a fixed 256-byte device array inside the library (64 ints, of which a call
 * uses 2), which every GPU that loads the library keeps until the process
 * exits.  One launch can hand out at most 2^31 - 1 work items (batch x heads
 * x groups of 4 query blocks); larger requests return LC_ERR_UNSUPPORTED.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress); make that first call before any stream capture.
 *   - All calls on a device share that device's array, which keeps the last
 *     call's contents; each call clears the counter on its stream before its
 *     kernel starts.  Calls on one device that overlap on the GPU (for
 *     example on two streams) race on the counter: serialise them.
 *   - In-kernel timeouts are reported by lc_last_device_status like the
 *     other entry points'.
 */
lc_status lc_bsa_forward_noalloc(const void *q, const void *k, const void *v, void *out,
                                 float *lse, int batch, int heads, int head_dim, lc_dtype dtype,
                                 float softmax_scale, lc_bsa_plan plan, lc_rope3d rope,
                                 void *stream);

/*
 * Context parallelism (myzaker / QbitAI "背后技术原理": block-sparse attention
 * is combined with context-parallel ring block-sparse attention for the
 * high-resolution pass).  The sequence's blocks are cut into contiguous
 * shards, one per rank; each rank keeps its query shard, the K/V shards
 * travel around a ring of ranks, and each step's partial result over one K/V
 * shard is merged into the rank's running result by log-sum-exp.  The pages
 * give no more than this; the pieces below are the device half of it (the
 * ring itself is the Python driver's send/recv over NCCL).
 *
 * lc_bsa_plan_create_shard -- the plan of lc_bsa_plan_create restricted to
 * query blocks [q_block_lo, q_block_hi) and key blocks [k_block_lo,
 * k_block_hi) (block ids as in lc_bsa_plan_create: condition blocks first).
 * The query bounds must be group boundaries: 0, multiples of 4 below Cb, Cb,
 * Cb + multiples of 4, or the block count (LC_ERR_INVALID_ARGUMENT
 * otherwise).  The key bounds are free.  A shard plan is accepted by
 * lc_bsa_forward_shard only; lc_bsa_plan_info reports its counts (nnz and
 * attended pairs of the shard) and lc_bsa_plan_copy_csr / _csc its entries.
 */
lc_status lc_bsa_plan_create_shard(lc_bsa_plan *out, int T, int H, int W, int block, int local,
                                   int stride, int n_cond_frames, int q_block_lo, int q_block_hi,
                                   int k_block_lo, int k_block_hi, void *stream);

/* Token ranges a plan covers: queries [*q_lo, *q_hi), keys [*k_lo, *k_hi)
 * (whole-sequence token indices; a full plan covers [0, N) twice). */
lc_status lc_bsa_plan_token_range(lc_bsa_plan plan, long long *q_lo, long long *q_hi,
                                  long long *k_lo, long long *k_hi);

/*
 * lc_bsa_forward_shard -- attention of the query tokens of a shard plan over
 * the key tokens of that plan only: q and out hold [batch, q_hi - q_lo,
 * heads, 64] (the plan's query token range, lc_bsa_plan_token_range), k and
 * v hold [batch, k_hi - k_lo, heads, 64] (pre-RoPE, like lc_bsa_forward's k;
 * they are rotated at their whole-sequence positions), lse (required) is
 * [batch, heads, q_hi - q_lo].  Rows that attend no key of the shard get
 * out = 0 and lse = -inf, so lc_bsa_lse_merge can take every shard's result
 * as it is.  opts: the RMSNorm weights of lc_bsa_forward_ex; flags
 * LC_FLAG_Q_ROTATED / LC_FLAG_K_ROTATED when q / k already hold the
 * normalised, rotated values (lc_rope3d_apply_ex at their whole-sequence
 * positions): a ring rotates each shard once and reuses it at every step.
 * The result is the same bits either way.  LC_FLAG_KEEP_EMPTY_ROWS: rows of
 * the plan's work groups (4 query blocks) that have no key in the shard are
 * not written, for a caller whose buffers already hold (0, -inf) there (the
 * set of such rows is fixed by the plan); rows of groups with keys are always
 * written, (0, -inf) included.  LC_FLAG_OVERLAP_PREVIOUS (needs
 * LC_FLAG_KEEP_EMPTY_ROWS): the launch is made with programmatic dependent
 * launch, so that its CTAs take the SMs the previous kernel on the stream
 * frees while that kernel's last work items finish, and its work-item
 * counter is the plan's own (reset by the kernel's last CTA) instead of one
 * set up by a memset between the launches.  The caller guarantees that this
 * launch reads nothing the previous kernel on the stream writes (true of the
 * steps of one ring rank: each writes its own out / lse, all read inputs
 * that were complete before the first step, which is made without the
 * flag), and that no other launch with the same plan is in flight.  The
 * kernel does not finish before the previous one, so a launch after it
 * without the flag sees every step's results.  bf16 only (LC_DTYPE_F32:
 * LC_ERR_UNSUPPORTED).  Errors as lc_bsa_forward.
 */
lc_status lc_bsa_forward_shard(const void *q, const void *k, const void *v, void *out, float *lse,
                               int batch, int heads, int head_dim, lc_dtype dtype,
                               float softmax_scale, const lc_bsa_opts *opts, lc_bsa_plan plan,
                               lc_rope3d rope, void *stream);

#define LC_MERGE_INIT 1u  /* the running result is not read: it starts as the part */

/*
 * lc_bsa_lse_merge -- fold one partial attention result (o_part of dtype,
 * lse_part fp32) into a running one (o_acc fp32, lse_acc fp32), per (batch,
 * token, head) row:  m = max(lse_acc, lse_part), w = e^(lse_acc - m),
 * w_p = e^(lse_part - m);  o = (w o_acc + w_p o_part) / (w + w_p),
 * lse = m + log(w + w_p); a row with both lse -inf stays (0, -inf).  The
 * result over a partition of the keys equals the attention over all of them.
 * Layouts: o_acc, o_part, out [batch, n_tokens, heads, 64]; lse_acc, lse_part
 * [batch, heads, n_tokens].  out NULL: o goes to o_acc; out given: o goes to
 * out, rounded to dtype, and o_acc is not written (the last step of a ring).
 * flags: LC_MERGE_INIT (o_acc and lse_acc not read; o_acc may then be NULL
 * when out is given).  lse_acc always receives the merged lse.  Errors:
 * LC_ERR_INVALID_ARGUMENT (NULL or misaligned pointer, bad sizes or flags),
 * LC_ERR_UNSUPPORTED (head_dim != 64, or more rows than one launch covers:
 * batch x n_tokens x heads x 8 threads past 2^31 - 1 blocks of 256).
 */
lc_status lc_bsa_lse_merge(float *o_acc, float *lse_acc, const void *o_part,
                           const float *lse_part, void *out, int batch, long long n_tokens,
                           int heads, int head_dim, lc_dtype dtype, unsigned flags, void *stream);

/*
 * lc_bsa_lse_merge_parts -- the merge of lc_bsa_lse_merge over n_parts
 * partial results at once: parts [n_parts, batch, n_tokens, heads, 64] of
 * dtype and lses [n_parts, batch, heads, n_tokens] fp32 (contiguous, part
 * after part) -> out [batch, n_tokens, heads, 64] of dtype and, if lse_out is
 * not NULL, lse_out [batch, heads, n_tokens]:  m = max_i lse_i,
 * w_i = e^(lse_i - m);  out = sum_i w_i o_i / sum_i w_i,
 * lse = m + log sum_i w_i (a row whose lse are all -inf: 0 and -inf).  One
 * pass, fp32 arithmetic, one rounding to dtype.  Errors: LC_ERR_INVALID_ARGUMENT
 * (NULL or misaligned pointer, n_parts <= 0, bad sizes), LC_ERR_UNSUPPORTED
 * (head_dim != 64, or more rows than one launch covers, as lc_bsa_lse_merge).
 */
lc_status lc_bsa_lse_merge_parts(const void *parts, const float *lses, int n_parts, void *out,
                                 float *lse_out, int batch, long long n_tokens, int heads,
                                 int head_dim, lc_dtype dtype, void *stream);

/*
 * lc_last_device_status -- synchronise `stream`, then report and clear the
 * current device's status word, which the kernels set when a bounded wait
 * timed out (LC_ERR_TIMEOUT) or an in-kernel check failed
 * (LC_ERR_DEVICE_CHECK).  LC_OK when nothing was flagged.
 */
lc_status lc_last_device_status(void *stream);

/*
 * lc_device_status_decode -- the status lc_last_device_status reports for a
 * device status word: bit 0 (a bounded in-kernel wait gave up) gives
 * LC_ERR_TIMEOUT, else bit 1 (an in-kernel check of the plan's lists failed:
 * a block id past the pattern, an empty member mask, a list bound outside
 * the plan's entries) gives LC_ERR_DEVICE_CHECK, else LC_OK.  Pure host
 * function, no CUDA call.
 */
lc_status lc_device_status_decode(int word);

/*
 * lc_debug_watchdog_selftest -- launch one CTA that waits, with the same
 * bounded wait the attention kernel uses, on a barrier that nothing ever
 * arrives on; the wait gives up after timeout_us microseconds and the kernel
 * returns normally.  Returns the device status that run left
 * (LC_ERR_TIMEOUT when the watchdog works).  For tests of failure detection.
 */
lc_status lc_debug_watchdog_selftest(int timeout_us, void *stream);

/*
 * lc_debug_scratch_pool_used_high -- the high-water mark, in bytes, of the
 * memory in use from the library's own scratch pool on the current device
 * (the stream-ordered pool the allocating entry points draw per-call scratch
 * from).  With reset != 0 the mark is first reset to the bytes in use now.
 * For tests that check which calls draw scratch (the allocation-free entry
 * point must not).  Synchronous; no GPU work.  Errors: LC_ERR_INVALID_ARGUMENT
 * when bytes is NULL, LC_ERR_CUDA when the pool cannot be reached.
 */
lc_status lc_debug_scratch_pool_used_high(unsigned long long *bytes, int reset);

/* Static description of a status code. */
const char *lc_status_string(lc_status s);

/* Library version, "major.minor.patch". */
const char *lc_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LC_BSA_H */
