// attn_bwd.cu -- backward pass of the block-sparse 3D-RoPE attention
// (gradients of q, k and v for the whole sequence), fp32 SIMT.
//
// Why: LongCat-Video is fine-tuned with LoRA adapters and gradient
// checkpointing (SimpleTuner page "Guia de Início Rápido do LongCat-Video
// Edit", section "2) Mudanças no config"), which needs this layer's input
// gradients.  What: the chain rule through the forward's definition, with the
// forward's lse (natural log) supplied by the caller:
//   p = exp(scale <q', k'> - lse),  D = <dO, O>,  ds = p (<dO, v> - D)
//   dq' = scale sum_k ds k',  dk' = scale sum_q ds q',  dv = sum_q p dO
//   dq = norm_q^T(R^T dq'),  dk = norm_k^T(R^T dk')
// with q' = R(norm_q(q)), R the partitioned 3D-RoPE ("longcat-video-rs",
// section 03-01) and the optional RMSNorm (myzaker / QbitAI "背后技术原理").
// The attended pairs are the plan's block pattern: dq walks a query block's
// CSR row, dk/dv walk a key block's CSC column ("longcat-video-rs", section
// 03-03).
//
// This file holds the fp32 path (bf16 goes to the tensor-core kernel in
// attn_bwd_sm100.cu) and the pieces both paths share.  Kernels: bwd_delta (D
// per row), bwd_dq (one CTA per query block x head x batch, one thread per
// query row, key blocks staged rotated in shared memory), bwd_dkdv (one CTA
// per key block, one thread per key row, query blocks staged),
// bwd_grad_finalize (dq, and dk under an RMSNorm, from the tensor-core
// path's fp32 sums).  Every rotation uses the library's shared pair routine and
// RMSNorm order, so q' and k' are the forward's values before rounding.
#include <cuda_bf16.h>
#include <math.h>
#include <string.h>

#include "lc_internal.cuh"
#include "lc_vec8.cuh"

namespace {

struct BwdArgs {
  const void *q, *k, *v, *o, *dout;
  const float *lse;
  float *delta;  // [B, heads, N] scratch
  void *dq, *dk, *dv;
  const int *row_ptr, *col_idx, *col_ptr, *row_idx;
  int *status;     // device status word (plan checks)
  long long nnz;   // CSR / CSC entries
  int n_blocks;    // blocks of the pattern
  const float *tab;
  const float *q_nw, *k_nw;
  float norm_eps, scale;
  int T, H, W;
  lc_divmod div_hw, div_w;
  int Nc, Nn, Cb, heads;
};

template <typename Tin>
__device__ __forceinline__ float ld(const Tin *p, long long i) {
  return (float)p[i];
}

template <typename Tin>
__device__ __forceinline__ void st(void *p, long long i, float x) {
  static_cast<Tin *>(p)[i] = (Tin)x;
}

// Row offset (in elements) of token n, head h, batch b of a [B, N, heads, 64] tensor.
__device__ __forceinline__ long long row_off(const BwdArgs &a, int b, int n, int h) {
  const long long N = (long long)a.Nc + a.Nn;
  return (((long long)b * N + n) * a.heads + h) * LC_HEAD_DIM;
}

// Tokens [lo, hi) of block id `blk` (condition blocks first).
__device__ __forceinline__ void block_range(const BwdArgs &a, int blk, int &lo, int &hi) {
  if (blk < a.Cb) {
    lo = LC_BLOCK * blk;
    hi = min(a.Nc, lo + LC_BLOCK);
  } else {
    lo = a.Nc + LC_BLOCK * (blk - a.Cb);
    hi = min(a.Nc + a.Nn, lo + LC_BLOCK);
  }
}

// Grid position of token n and the cos / sin of its pair p (0..31).
struct Pos {
  int t, hh, w;
};
__device__ __forceinline__ Pos decode(const BwdArgs &a, int n) {
  Pos q;
  q.t = lc_div(n, a.div_hw);
  const int rem = n - q.t * a.div_hw.d;
  q.hh = lc_div(rem, a.div_w);
  q.w = rem - q.hh * a.div_w.d;
  return q;
}
__device__ __forceinline__ void pair_angle(const BwdArgs &a, const Pos &q, int p, float &c,
                                           float &s) {
  const float *tab = a.tab;
  if (p < 8) {
    c = __ldg(tab + q.t * 8 + p);
    s = __ldg(tab + a.T * 8 + q.t * 8 + p);
  } else if (p < 20) {
    c = __ldg(tab + a.T * 16 + q.hh * 12 + p - 8);
    s = __ldg(tab + a.T * 16 + a.H * 12 + q.hh * 12 + p - 8);
  } else {
    c = __ldg(tab + a.T * 16 + a.H * 24 + q.w * 12 + p - 20);
    s = __ldg(tab + a.T * 16 + a.H * 24 + a.W * 12 + q.w * 12 + p - 20);
  }
}

// 1 / rms of a 64-channel row, summed in the library's fixed order.
__device__ __forceinline__ float row_rms_inv(const float *x, float eps) {
  float c8[8];
#pragma unroll
  for (int ch = 0; ch < 8; ++ch) c8[ch] = lc_sumsq8(x + 8 * ch);
  return lc_rms_inv(lc_sumsq_tree8(c8), eps);
}

// x <- R(norm(x)) for token n (the forward's q' / k').
__device__ __forceinline__ void norm_rotate(const BwdArgs &a, float *x, int n, const float *nw) {
  if (nw) {
    const float inv = row_rms_inv(x, a.norm_eps);
#pragma unroll
    for (int d = 0; d < LC_HEAD_DIM; ++d) x[d] = lc_rms_apply(x[d], inv, __ldg(nw + d));
  }
  const Pos pos = decode(a, n);
#pragma unroll
  for (int p = 0; p < 32; ++p) {
    float c, s;
    pair_angle(a, pos, p, c, s);
    lc_rot_pair(x[2 * p], x[2 * p + 1], c, s, x[2 * p], x[2 * p + 1]);
  }
}

// g <- norm^T(R^T g) for token n; x is the raw (pre-norm) input row.
__device__ __forceinline__ void rotate_norm_transpose(const BwdArgs &a, float *g, const float *x,
                                                      int n, const float *nw) {
  const Pos pos = decode(a, n);
#pragma unroll
  for (int p = 0; p < 32; ++p) {  // R^T: turn each pair back
    float c, s;
    pair_angle(a, pos, p, c, s);
    const float u = g[2 * p], w = g[2 * p + 1];
    g[2 * p] = fmaf(u, c, w * s);
    g[2 * p + 1] = fmaf(w, c, -u * s);
  }
  if (nw) {  // y = x inv w:  dx = inv (w g) - x inv^3 / 64 * sum(g w x)
    const float inv = row_rms_inv(x, a.norm_eps);
    float dot = 0.f;
#pragma unroll
    for (int d = 0; d < LC_HEAD_DIM; ++d) dot = fmaf(g[d] * __ldg(nw + d), x[d], dot);
    const float k3 = inv * inv * inv * (1.f / LC_HEAD_DIM) * dot;
#pragma unroll
    for (int d = 0; d < LC_HEAD_DIM; ++d) g[d] = inv * __ldg(nw + d) * g[d] - x[d] * k3;
  }
}

using lcvec::ld8;
using lcvec::st8;

// D[b, h, n] = <dO_n, O_n>; eight lanes per (batch, token, head) row, each
// on one 8-channel chunk (coalesced vector loads), combined by shuffles.
template <typename Tin>
__global__ void bwd_delta_kernel(BwdArgs a, long long rows) {
  const long long gid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  const long long i = gid >> 3;
  const int ch = (int)(gid & 7);
  if (i >= rows) return;  // rows are whole 8-lane groups: the group leaves together
  const unsigned group = 0xFFu << (threadIdx.x & 24);
  float o[8], g[8];
  ld8(static_cast<const Tin *>(a.o) + i * LC_HEAD_DIM + 8 * ch, o);
  ld8(static_cast<const Tin *>(a.dout) + i * LC_HEAD_DIM + 8 * ch, g);
  float acc = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) acc = fmaf(o[e], g[e], acc);
  acc += __shfl_xor_sync(group, acc, 1);
  acc += __shfl_xor_sync(group, acc, 2);
  acc += __shfl_xor_sync(group, acc, 4);
  if (ch == 0) {
    const int h = (int)(i % a.heads);
    const long long bn = i / a.heads;  // b * N + n
    const long long N = (long long)a.Nc + a.Nn;
    const int n = (int)(bn % N), b = (int)(bn / N);
    a.delta[((long long)b * a.heads + h) * N + n] = acc;
  }
}

// Shared memory rows are padded to 65 floats: a thread walking its own row
// and a warp reading one row broadcast are both free of bank conflicts.
constexpr int kRow = LC_HEAD_DIM + 1;
constexpr size_t kBwdSmem = 4 * LC_BLOCK * kRow * sizeof(float) + 2 * LC_BLOCK * sizeof(float);

// One CTA per (query block, head, batch); thread = query row.  The thread's
// own q' and dO rows live in shared memory; dq' accumulates in registers.
template <typename Tin>
__global__ void __launch_bounds__(64) bwd_dq_kernel(BwdArgs a) {
  extern __shared__ float smem[];
  float(*sK)[kRow] = reinterpret_cast<float(*)[kRow]>(smem);
  float(*sV)[kRow] = sK + LC_BLOCK;
  float(*sQm)[kRow] = sV + LC_BLOCK;
  float(*sGm)[kRow] = sQm + LC_BLOCK;
  const int r = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const long long N = (long long)a.Nc + a.Nn;
  int q_lo, q_hi;
  block_range(a, r, q_lo, q_hi);
  const int n = q_lo + tid;
  const bool valid = n < q_hi;
  const Tin *Q = static_cast<const Tin *>(a.q);
  const Tin *G = static_cast<const Tin *>(a.dout);
  float lse = 0.f, delta = 0.f;
  if (valid) {
    const long long off = row_off(a, b, n, h);
    for (int d = 0; d < LC_HEAD_DIM; ++d) {
      sQm[tid][d] = ld(Q, off + d);
      sGm[tid][d] = ld(G, off + d);
    }
    norm_rotate(a, sQm[tid], n, a.q_nw);
    lse = a.lse[((long long)b * a.heads + h) * N + n];
    delta = a.delta[((long long)b * a.heads + h) * N + n];
  }
  float dq[LC_HEAD_DIM];
#pragma unroll
  for (int d = 0; d < LC_HEAD_DIM; ++d) dq[d] = 0.f;
  const Tin *K = static_cast<const Tin *>(a.k);
  const Tin *V = static_cast<const Tin *>(a.v);
  int e_lo, e_hi;
  lc_checked_row(a.row_ptr, r, a.nnz, a.status, e_lo, e_hi);
  for (int e = e_lo; e < e_hi; ++e) {
    if (!lc_checked_block(a.col_idx[e], a.n_blocks, a.status)) continue;
    int k_lo, k_hi;
    block_range(a, a.col_idx[e], k_lo, k_hi);
    const int kn = k_hi - k_lo;
    __syncthreads();
    if (tid < kn) {  // each thread stages one key row, rotated in place
      const int m = k_lo + tid;
      const long long off = row_off(a, b, m, h);
      for (int d = 0; d < LC_HEAD_DIM; ++d) {
        sK[tid][d] = ld(K, off + d);
        sV[tid][d] = ld(V, off + d);
      }
      norm_rotate(a, sK[tid], m, a.k_nw);
    }
    __syncthreads();
    if (valid) {
      for (int j = 0; j < kn; ++j) {
        float s = 0.f, dp = 0.f;
#pragma unroll 16
        for (int d = 0; d < LC_HEAD_DIM; ++d) {
          s = fmaf(sQm[tid][d], sK[j][d], s);
          dp = fmaf(sGm[tid][d], sV[j][d], dp);
        }
        const float p = expf(a.scale * s - lse);
        const float ds = a.scale * p * (dp - delta);
#pragma unroll
        for (int d = 0; d < LC_HEAD_DIM; ++d) dq[d] = fmaf(ds, sK[j][d], dq[d]);
      }
    }
  }
  if (!valid) return;
  const long long off = row_off(a, b, n, h);
  for (int d = 0; d < LC_HEAD_DIM; ++d) sQm[tid][d] = ld(Q, off + d);  // raw row for the norm
  rotate_norm_transpose(a, dq, sQm[tid], n, a.q_nw);
#pragma unroll
  for (int d = 0; d < LC_HEAD_DIM; ++d) st<Tin>(a.dq, off + d, dq[d]);
}

// One CTA per (key block, head, batch); thread = key row.  Its own k' and v
// rows live in shared memory; dk' and dv accumulate in registers.
template <typename Tin>
__global__ void __launch_bounds__(64) bwd_dkdv_kernel(BwdArgs a) {
  extern __shared__ float smem[];
  float(*sQ)[kRow] = reinterpret_cast<float(*)[kRow]>(smem);  // staged query block, rotated
  float(*sG)[kRow] = sQ + LC_BLOCK;                            // its dO
  float(*sKm)[kRow] = sG + LC_BLOCK;                           // this CTA's rotated keys
  float(*sVm)[kRow] = sKm + LC_BLOCK;                          // and values
  float *sL = smem + 4 * LC_BLOCK * kRow, *sD = sL + LC_BLOCK;
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const long long N = (long long)a.Nc + a.Nn;
  int k_lo, k_hi;
  block_range(a, c, k_lo, k_hi);
  const int m = k_lo + tid;
  const bool valid = m < k_hi;
  const Tin *K = static_cast<const Tin *>(a.k);
  const Tin *V = static_cast<const Tin *>(a.v);
  if (valid) {
    const long long off = row_off(a, b, m, h);
    for (int d = 0; d < LC_HEAD_DIM; ++d) {
      sKm[tid][d] = ld(K, off + d);
      sVm[tid][d] = ld(V, off + d);
    }
    norm_rotate(a, sKm[tid], m, a.k_nw);
  }
  float dk[LC_HEAD_DIM], dv[LC_HEAD_DIM];
#pragma unroll
  for (int d = 0; d < LC_HEAD_DIM; ++d) dk[d] = dv[d] = 0.f;
  const Tin *Q = static_cast<const Tin *>(a.q);
  const Tin *G = static_cast<const Tin *>(a.dout);
  int e_lo, e_hi;
  lc_checked_row(a.col_ptr, c, a.nnz, a.status, e_lo, e_hi);
  for (int e = e_lo; e < e_hi; ++e) {
    if (!lc_checked_block(a.row_idx[e], a.n_blocks, a.status)) continue;
    int q_lo, q_hi;
    block_range(a, a.row_idx[e], q_lo, q_hi);
    const int qn = q_hi - q_lo;
    __syncthreads();
    if (tid < qn) {  // each thread stages one query row, rotated in place
      const int n = q_lo + tid;
      const long long off = row_off(a, b, n, h);
      for (int d = 0; d < LC_HEAD_DIM; ++d) {
        sQ[tid][d] = ld(Q, off + d);
        sG[tid][d] = ld(G, off + d);
      }
      norm_rotate(a, sQ[tid], n, a.q_nw);
      sL[tid] = a.lse[((long long)b * a.heads + h) * N + n];
      sD[tid] = a.delta[((long long)b * a.heads + h) * N + n];
    }
    __syncthreads();
    if (valid) {
      for (int i = 0; i < qn; ++i) {
        float s = 0.f, dp = 0.f;
#pragma unroll 16
        for (int d = 0; d < LC_HEAD_DIM; ++d) {
          s = fmaf(sQ[i][d], sKm[tid][d], s);
          dp = fmaf(sG[i][d], sVm[tid][d], dp);
        }
        const float p = expf(a.scale * s - sL[i]);
        const float ds = a.scale * p * (dp - sD[i]);
#pragma unroll
        for (int d = 0; d < LC_HEAD_DIM; ++d) {
          dv[d] = fmaf(p, sG[i][d], dv[d]);
          dk[d] = fmaf(ds, sQ[i][d], dk[d]);
        }
      }
    }
  }
  if (!valid) return;
  const long long off = row_off(a, b, m, h);
  for (int d = 0; d < LC_HEAD_DIM; ++d) sKm[tid][d] = ld(K, off + d);  // raw row for the norm
  rotate_norm_transpose(a, dk, sKm[tid], m, a.k_nw);
#pragma unroll
  for (int d = 0; d < LC_HEAD_DIM; ++d) {
    st<Tin>(a.dk, off + d, dk[d]);
    st<Tin>(a.dv, off + d, dv[d]);
  }
}

// g = norm^T(R^T acc) per (batch, token, head) row: dq from the tensor-core
// path's fp32 dq sums (raw rows = q, weights = q's), or dk from its fp32 dk'
// when k is normalised (raw rows = k).  Eight lanes per row, one 8-channel
// chunk (4 RoPE pairs) each; the norm's row sums by shuffles.
template <typename Tin>
__global__ void bwd_grad_finalize_kernel(BwdArgs a, const float *acc, long long rows) {
  const long long gid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  const long long i = gid >> 3;
  const int ch = (int)(gid & 7);
  if (i >= rows) return;  // rows are whole 8-lane groups: the group leaves together
  const unsigned group = 0xFFu << (threadIdx.x & 24);
  const long long N = (long long)a.Nc + a.Nn;
  const int n = (int)((i / a.heads) % N);
  float g[8];
  ld8(acc + i * LC_HEAD_DIM + 8 * ch, g);
  const Pos pos = decode(a, n);
#pragma unroll
  for (int q2 = 0; q2 < 4; ++q2) {  // R^T: turn each pair back
    float c, sn;
    pair_angle(a, pos, 4 * ch + q2, c, sn);
    const float u = g[2 * q2], w = g[2 * q2 + 1];
    g[2 * q2] = fmaf(u, c, w * sn);
    g[2 * q2 + 1] = fmaf(w, c, -u * sn);
  }
  if (a.q_nw) {  // y = x inv w:  dx = inv (w g) - x inv^3 / 64 * sum(g w x)
    float x[8], w8[8];
    ld8(static_cast<const Tin *>(a.q) + i * LC_HEAD_DIM + 8 * ch, x);
#pragma unroll
    for (int e = 0; e < 8; ++e) w8[e] = __ldg(a.q_nw + 8 * ch + e);
    const float inv = lc_rms_inv(lc_sumsq_lanes8(lc_sumsq8(x), group), a.norm_eps);
    float dot = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) dot = fmaf(g[e] * w8[e], x[e], dot);
    dot += __shfl_xor_sync(group, dot, 1);
    dot += __shfl_xor_sync(group, dot, 2);
    dot += __shfl_xor_sync(group, dot, 4);
    const float k3 = inv * inv * inv * (1.f / LC_HEAD_DIM) * dot;
#pragma unroll
    for (int e = 0; e < 8; ++e) g[e] = inv * w8[e] * g[e] - x[e] * k3;
  }
  st8(static_cast<Tin *>(a.dq) + i * LC_HEAD_DIM + 8 * ch, g);
}

template <typename Tin>
lc_status launch_all(const BwdArgs &a, int batch, int nq, cudaStream_t st) {
  const long long rows = (long long)batch * (a.Nc + a.Nn) * a.heads;
  bwd_delta_kernel<Tin><<<(unsigned)((rows * 8 + 255) / 256), 256, 0, st>>>(a, rows);
  dim3 grid(nq, a.heads, batch);
  LC_CUDA_TRY(cudaFuncSetAttribute(bwd_dq_kernel<Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)kBwdSmem));
  LC_CUDA_TRY(cudaFuncSetAttribute(bwd_dkdv_kernel<Tin>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kBwdSmem));
  bwd_dq_kernel<Tin><<<grid, 64, kBwdSmem, st>>>(a);
  bwd_dkdv_kernel<Tin><<<grid, 64, kBwdSmem, st>>>(a);
  return lc_from_cuda(cudaGetLastError());
}

}  // namespace

lc_status lc_bwd_delta(const void *out, const void *dout, float *delta, int batch, long long N,
                       int heads, lc_dtype dtype, cudaStream_t stream) {
  BwdArgs a;
  memset(&a, 0, sizeof(a));
  a.o = out; a.dout = dout; a.delta = delta; a.heads = heads;
  a.Nc = 0; a.Nn = (int)N;
  const long long rows = (long long)batch * N * heads;
  if (rows == 0) return LC_OK;
  const unsigned grid = (unsigned)((rows * 8 + 255) / 256);  // 8 lanes per row
  if (dtype == LC_DTYPE_F32)
    bwd_delta_kernel<float><<<grid, 256, 0, stream>>>(a, rows);
  else
    bwd_delta_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(a, rows);
  return lc_from_cuda(cudaGetLastError());
}

lc_status lc_bwd_grad_finalize(const float *acc, const void *raw, void *grad, int batch,
                               long long N, int heads, lc_dtype dtype, const float *nw, float eps,
                               const lc_rope3d_s *rope, cudaStream_t stream) {
  BwdArgs a;
  memset(&a, 0, sizeof(a));
  a.q = raw; a.dq = grad; a.heads = heads; a.Nc = 0; a.Nn = (int)N;
  a.tab = rope->tab;
  a.q_nw = nw; a.norm_eps = eps;
  a.T = rope->T; a.H = rope->H; a.W = rope->W;
  a.div_hw = lc_make_divmod(rope->H * rope->W);
  a.div_w = lc_make_divmod(rope->W);
  const long long rows = (long long)batch * N * heads;
  if (rows == 0) return LC_OK;
  const unsigned grid = (unsigned)((rows * 8 + 255) / 256);  // 8 lanes per row
  if (dtype == LC_DTYPE_F32)
    bwd_grad_finalize_kernel<float><<<grid, 256, 0, stream>>>(a, acc, rows);
  else
    bwd_grad_finalize_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(a, acc, rows);
  return lc_from_cuda(cudaGetLastError());
}

lc_status lc_launch_backward(const void *q, const void *k, const void *v, const void *out,
                             const float *lse, const void *dout, void *dq, void *dk, void *dv,
                             int batch, int heads, float scale, lc_dtype dtype,
                             const lc_qk_norm &norm, const lc_bsa_plan_s *plan,
                             const lc_rope3d_s *rope, cudaStream_t stream) {
  if (dtype == LC_DTYPE_BF16)  // the tensor-core path
    return lc_launch_backward_sm100(q, k, v, out, lse, dout, dq, dk, dv, batch, heads, scale,
                                    norm, plan, rope, stream);
  BwdArgs a;
  a.q = q; a.k = k; a.v = v; a.o = out; a.dout = dout; a.lse = lse;
  a.dq = dq; a.dk = dk; a.dv = dv;
  a.row_ptr = plan->row_ptr; a.col_idx = plan->col_idx;
  a.col_ptr = plan->col_ptr; a.row_idx = plan->row_idx;
  a.nnz = plan->nnz;
  a.n_blocks = plan->Cb + plan->Nb;
  a.tab = rope->tab;
  a.q_nw = norm.q_w; a.k_nw = norm.k_w; a.norm_eps = norm.eps;
  a.scale = scale;
  a.T = rope->T; a.H = rope->H; a.W = rope->W;
  a.div_hw = lc_make_divmod(rope->H * rope->W);
  a.div_w = lc_make_divmod(rope->W);
  a.Nc = plan->Nc; a.Nn = plan->Nn; a.Cb = plan->Cb; a.heads = heads;
  if (plan->nq == 0) return LC_OK;
  lc_status s = LC_OK;
  a.status = lc_device_status_ptr(&s);
  if (s != LC_OK) return s;
  cudaMemPool_t pool = lc_scratch_pool(&s);
  if (s != LC_OK) return s;
  const size_t dbytes = sizeof(float) * (size_t)batch * heads * (plan->Nc + plan->Nn);
  float *delta = nullptr;
  LC_CUDA_TRY(cudaStreamWaitEvent(stream, plan->ready, 0));
  LC_CUDA_TRY(cudaStreamWaitEvent(stream, rope->ready, 0));
  cudaError_t e = cudaMallocFromPoolAsync(reinterpret_cast<void **>(&delta), dbytes, pool, stream);
  if (e != cudaSuccess) return lc_from_cuda(e);
  a.delta = delta;
  s = launch_all<float>(a, batch, plan->nq, stream);
  cudaFreeAsync(delta, stream);
  return s;
}
