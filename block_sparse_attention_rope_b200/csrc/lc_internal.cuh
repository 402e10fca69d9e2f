// lc_internal.cuh -- definitions shared by the translation units of liblcbsa.so
// (plan and rope handles, status plumbing, launch helpers).  Not installed.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/lc_bsa.h"

// Device status bits written by kernels (see lc_last_device_status).
#define LC_DEVSTAT_TIMEOUT 0x1
#define LC_DEVSTAT_CHECK 0x2

#ifdef __CUDACC__
// One row [lo, hi) of a plan's CSR (or CSC) lists with its bounds checked: a
// row that a consistent plan never holds (negative, reversed, or past the
// nnz entries) is walked as an empty row and LC_DEVSTAT_CHECK is raised.
__device__ __forceinline__ void lc_checked_row(const int *ptr, int r, long long nnz, int *status,
                                               int &lo, int &hi) {
  lo = ptr[r];
  hi = ptr[r + 1];
  if (lo < 0 || hi < lo || (long long)hi > nnz) {
    if (status && threadIdx.x == 0) atomicOr(status, LC_DEVSTAT_CHECK);
    lo = hi = 0;
  }
}
// A block id of a list entry, checked against the pattern's block count; the
// caller skips the entry when this returns false (LC_DEVSTAT_CHECK raised).
__device__ __forceinline__ bool lc_checked_block(int c, int n_blocks, int *status) {
  if ((unsigned)c < (unsigned)n_blocks) return true;
  if (status && threadIdx.x == 0) atomicOr(status, LC_DEVSTAT_CHECK);
  return false;
}
#endif

// Tokens of one block, head dimension and RoPE split supported by v1.
#define LC_BLOCK 64
#define LC_HEAD_DIM 64

// Block-sparse plan.  All arrays live in one device allocation `mem`.
//
// Block ids: 0..Cb-1 are condition blocks (tokens [64c, min(Nc, 64c+64)) of the
// condition segment), Cb..Cb+Nb-1 noisy blocks (tokens [64j, ...) of the noisy
// segment).  A "group" is up to 4 consecutive query blocks of one segment,
// the unit of work of the tensor-core kernel (two 128-row query tiles); its
// entry list is the sorted union of its members' key blocks, each entry
// holding (key block id) | (member mask << 24).
struct lc_bsa_plan_s {
  int T, H, W, block, local, stride, n_cond;
  int Nc, Nn, Cb, Nb, nq;
  int gc, gn, G;            // groups in the condition / noisy segment, total
  int qlo, qhi, klo, khi;   // block ranges the plan covers (a shard plan: part of the pattern)
  int G_active;             // groups with at least one entry (the first G_active of grp_order)
  bool fill_needed;         // a group of the query range has no entry (shard plans)
  long long nnz;            // CSR entries (host closed form, checked on device)
  int device;
  cudaEvent_t ready;        // recorded after the planner kernels
  void *mem;
  int *row_ptr;             // [nq + 1]
  int *col_idx;             // [nnz]
  int *row_cnt;             // [nq]      planner work array
  int *grp_ptr;             // [G + 1]
  int *grp_cnt;             // [G]       planner work array
  uint32_t *grp_ent;        // [nnz]     (upper bound of the union lists)
  int *grp_order;           // [G]       groups by entry count, longest first
  int *col_ptr;             // [nq + 1]  transpose (CSC): query blocks attending key block c
  int *row_idx;             // [nnz]     ascending
  int *col_cnt;             // [nq]      planner work array
  // Backward work lists: key groups of up to 2 key blocks of one segment
  // with alike query lists (kgc condition groups, then kgn noisy ones; see
  // kgroup_members in plan.cu), each with the sorted
  // union of the query blocks attending either member (entry = query block id
  // | member mask << 24), and the groups ranked longest list first.
  int kgc, kgn, KG;
  int *kgrp_ptr;            // [KG + 1]
  int *kgrp_cnt;            // [KG]
  uint32_t *kgrp_ent;       // [nnz]     (upper bound of the union lists)
  int *kgrp_order;          // [KG]
  int2 *kgrp_blk;           // [KG]      the group's key blocks (second -1 if none)
  unsigned long long *pairs;  // [2] attended token pairs: all rows, noisy rows
  int *err;                 // [1] planner consistency flag
  int *sched;               // [2] work-item and finished-CTA counters of launches that use
                            //     the plan's own scheduler (zero between launches)
  long long pairs_host[2];
  bool info_cached;
};

// A plan restricted to part of the pattern (lc_bsa_plan_create_shard).
inline bool lc_plan_is_shard(const lc_bsa_plan_s *p) {
  return p->qlo != 0 || p->qhi != p->nq || p->klo != 0 || p->khi != p->nq;
}
// First token of block r in the whole sequence (r == nq: the token count).
inline long long lc_block_token(const lc_bsa_plan_s *p, int r) {
  const long long t = r < p->Cb ? (long long)LC_BLOCK * r
                                : (long long)p->Nc + (long long)LC_BLOCK * (r - p->Cb);
  const long long n = (long long)p->Nc + p->Nn;
  return t < n ? t : n;
}

// RoPE tables: fp32 [cos_t T*dt/2][sin_t][cos_h H*dh/2][sin_h][cos_w W*dw/2][sin_w].
struct lc_rope3d_s {
  int T, H, W;
  double theta;
  int dt, dh, dw;
  int device;
  cudaEvent_t ready;        // recorded after the table kernel
  long long n_floats;
  float *tab;
};

// Per-device library state: the status word kernels report into, and the
// library's stream-ordered pool for per-call scratch (keeps its memory).
int *lc_device_status_ptr(lc_status *st);
cudaMemPool_t lc_scratch_pool(lc_status *st);

// Map a CUDA error to a status (out-of-memory gets its own code).
static inline lc_status lc_from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return LC_OK;
  if (e == cudaErrorMemoryAllocation) return LC_ERR_OUT_OF_MEMORY;
  return LC_ERR_CUDA;
}

#define LC_CUDA_TRY(expr)                                   \
  do {                                                      \
    cudaError_t _e = (expr);                                \
    if (_e != cudaSuccess) return lc_from_cuda(_e);         \
  } while (0)

// Fast exact division of non-negative n < 2^24 by a constant d < 2^16:
// q = (n * m) >> 40 with m = ceil(2^40 / d).  Exact because the rounding
// error n*(m*d - 2^40) < n*d <= 2^40 keeps the quotient's integer part.
struct lc_divmod {
  unsigned long long m;
  int d;
};
static inline lc_divmod lc_make_divmod(int d) {
  lc_divmod r;
  r.d = d;
  r.m = ((1ull << 40) + (unsigned long long)d - 1ull) / (unsigned long long)d;
  return r;
}
__device__ __forceinline__ int lc_div(int n, lc_divmod dm) {
  return (int)(((unsigned long long)(unsigned)n * dm.m) >> 40);
}

// One RoPE channel pair (a, b) rotated by the angle with cosine c and sine s:
// (a c - b s, a s + b c), each as one rounded product and one fused
// multiply-add, spelled out so that every kernel that rotates (Q and K tiles,
// the K pass, the public rotation, the fp32 path) produces the same bits for
// the same input whatever the compiler would contract.
__device__ __forceinline__ void lc_rot_pair(float a, float b, float c, float s, float &x,
                                            float &y) {
  x = __fmaf_rn(a, c, -__fmul_rn(b, s));
  y = __fmaf_rn(a, s, __fmul_rn(b, c));
}

// RMSNorm of one 64-channel row (one token, one head) ahead of the rotation
// (myzaker / QbitAI "背后技术原理": RMSNorm in the attention modules):
// y = x / sqrt(mean(x^2) + eps) * w.  The mean square is summed in a fixed
// order -- each 8-channel chunk sequentially, then the eight chunk sums as
// ((c0+c1)+(c2+c3))+((c4+c5)+(c6+c7)) -- so that a thread holding the whole
// row and eight lanes holding one chunk each (combined by xor-shuffles over
// 1, 2, 4, which form the same sums) get the same bits.
__device__ __forceinline__ float lc_sumsq8(const float *x) {
  float a = __fmul_rn(x[0], x[0]);
#pragma unroll
  for (int i = 1; i < 8; ++i) a = __fmaf_rn(x[i], x[i], a);
  return a;
}
__device__ __forceinline__ float lc_sumsq_tree8(const float *c) {
  return __fadd_rn(__fadd_rn(__fadd_rn(c[0], c[1]), __fadd_rn(c[2], c[3])),
                   __fadd_rn(__fadd_rn(c[4], c[5]), __fadd_rn(c[6], c[7])));
}
// Eight consecutive lanes (mask: their bits) each hold one chunk sum.
__device__ __forceinline__ float lc_sumsq_lanes8(float c, unsigned mask) {
  c = __fadd_rn(c, __shfl_xor_sync(mask, c, 1));
  c = __fadd_rn(c, __shfl_xor_sync(mask, c, 2));
  return __fadd_rn(c, __shfl_xor_sync(mask, c, 4));
}
__device__ __forceinline__ float lc_rms_inv(float sumsq, float eps) {
  return rsqrtf(__fmaf_rn(sumsq, 0.015625f, eps));  // mean = sum / 64
}
__device__ __forceinline__ float lc_rms_apply(float x, float inv, float w) {
  return __fmul_rn(__fmul_rn(x, inv), w);
}

// Launch helpers implemented by the kernel translation units.
// Which queries an attention launch computes and where its tensors live.
//   LC_FWD_FULL    q, k, v, out hold all N tokens (cond_k / cond_v unused).
//   LC_FWD_CACHED  q, k, v, out hold the Nn noisy tokens; the condition
//                  tokens' K/V come from cond_k / cond_v ([B, Nc, heads, 64]).
//   LC_FWD_COND    only the condition queries: q and out hold the Nc condition
//                  tokens, K/V come from cond_k / cond_v (k and v unused).
//   LC_FWD_SHARD   one shard of the whole-sequence attention (context
//                  parallelism): q and out hold tokens [q_lo, q_lo + q_n), k
//                  and v tokens [k_lo, k_lo + k_n) (lc_shard_view); the plan
//                  is a shard plan over those blocks (bf16 only).
// cond_k_rotated: cond_k already holds R(k) (CACHED and COND only).
enum lc_fwd_mode { LC_FWD_FULL = 0, LC_FWD_CACHED = 1, LC_FWD_COND = 2, LC_FWD_SHARD = 3 };
struct lc_shard_view {
  long long q_lo, q_n, k_lo, k_n;
  bool q_rotated, k_rotated;  // q / k already hold R(norm(x)) (rotated once per ring)
  bool overlap_previous;      // programmatic dependent launch, the plan's own scheduler
};

// RMSNorm of q and k ahead of the rotation: device fp32 weights [64] or NULL.
struct lc_qk_norm {
  const float *q_w = nullptr;
  const float *k_w = nullptr;
  float eps = 0.f;
};

lc_status lc_launch_forward_f32(const float *q, const float *k, const float *v,
                                const float *cond_k, const float *cond_v, float *out,
                                float *lse, int batch, int heads, float scale, lc_fwd_mode mode,
                                bool cond_k_rotated, const lc_qk_norm &norm,
                                const lc_bsa_plan_s *plan, const lc_rope3d_s *rope,
                                int *dev_status, cudaStream_t stream);
// counter_scratch: NULL = allocate the scheduler counter stream-ordered for
// this launch; else a device int the caller provides (lc_bsa_forward_noalloc,
// LC_FWD_FULL only).
lc_status lc_launch_forward_sm100(const void *q, const void *k, const void *v,
                                  const void *cond_k, const void *cond_v, void *out,
                                  float *lse, int batch, int heads, float scale, lc_fwd_mode mode,
                                  bool cond_k_rotated, const lc_qk_norm &norm,
                                  const lc_bsa_plan_s *plan, const lc_rope3d_s *rope,
                                  int *dev_status, cudaStream_t stream,
                                  int *counter_scratch = nullptr,
                                  const lc_shard_view *shard = nullptr);
// Context parallelism pieces (ring.cu): rows of a shard plan's query range
// that no launch writes (groups without entries) get out = 0, lse = -inf;
// the online-softmax merge of a partial result into a running one.
lc_status lc_launch_shard_fill(const lc_bsa_plan_s *plan, void *out, float *lse, int batch,
                               int heads, lc_dtype dtype, cudaStream_t stream);
lc_status lc_launch_lse_merge(float *o_acc, float *lse_acc, const void *o_part,
                              const float *lse_part, void *out, int batch, long long n, int heads,
                              lc_dtype dtype, bool init, cudaStream_t stream);
lc_status lc_launch_lse_merge_parts(const void *parts, const float *lses, int n_parts, void *out,
                                    float *lse_out, int batch, long long n, int heads,
                                    lc_dtype dtype, cudaStream_t stream);
// Gradients dq, dk, dv of the whole-sequence attention (attn_bwd.cu).
lc_status lc_launch_backward(const void *q, const void *k, const void *v, const void *out,
                             const float *lse, const void *dout, void *dq, void *dk, void *dv,
                             int batch, int heads, float scale, lc_dtype dtype,
                             const lc_qk_norm &norm, const lc_bsa_plan_s *plan,
                             const lc_rope3d_s *rope, cudaStream_t stream);
// The tensor-core backward (attn_bwd_sm100.cu, bf16), and the pieces of the
// backward shared by both paths (attn_bwd.cu): D = rowsum(dO * O) per row, and
// grad = norm^T(R^T acc) cast to dtype (dq; dk under an RMSNorm).
lc_status lc_launch_backward_sm100(const void *q, const void *k, const void *v, const void *out,
                                   const float *lse, const void *dout, void *dq, void *dk,
                                   void *dv, int batch, int heads, float scale,
                                   const lc_qk_norm &norm, const lc_bsa_plan_s *plan,
                                   const lc_rope3d_s *rope, cudaStream_t stream);
// R(norm(x)) of a bf16 [batch, ntok, heads, 64] tensor into dst, with the
// attention kernels' exact arithmetic (attn_sm100.cu).
lc_status lc_rope_rows_bf16(const void *src, void *dst, int batch, long long ntok, int heads,
                            int tok_offset, const lc_rope3d_s *rope, const float *nw, float eps,
                            cudaStream_t stream);
lc_status lc_bwd_delta(const void *out, const void *dout, float *delta, int batch, long long N,
                       int heads, lc_dtype dtype, cudaStream_t stream);
lc_status lc_bwd_grad_finalize(const float *acc, const void *raw, void *grad, int batch,
                               long long N, int heads, lc_dtype dtype, const float *nw, float eps,
                               const lc_rope3d_s *rope, cudaStream_t stream);
// Rotate x [batch, ntok, heads, 64] of dtype (token n of x = sequence token
// n + tok_offset) into out, after an RMSNorm with norm_w when not NULL
// (rope.cu; the public lc_rope3d_apply is this without the norm).  Arguments
// are checked by the caller.
lc_status lc_rotate_rows(const void *x, void *out, int batch, long long ntok, int heads,
                         long long tok_offset, lc_dtype dtype, const lc_rope3d_s *rope,
                         const float *norm_w, float eps, cudaStream_t stream);

// Fixed scratch of lc_bsa_forward_noalloc (attn_sm100.cu): device address of
// g_lc_noalloc_scratch on the current device, looked up once per device.
#define LC_NOALLOC_SCRATCH_INTS 64
int *lc_noalloc_scratch(lc_status *st);
// The same address if it has been looked up on the current device already,
// else NULL (no lookup, no CUDA call beyond cudaGetDevice).
int *lc_noalloc_scratch_if_ready();
lc_status lc_launch_watchdog_selftest(int *dev_status, long long timeout_ns, cudaStream_t stream);
