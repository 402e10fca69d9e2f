// attn_f32.cu -- fp32 SIMT block-sparse 3D-RoPE attention.
//
// One CTA per (query block, head, batch), one thread per query row.  The CTA
// walks the query block's key-block list (the plan's CSR row), stages each key
// block in shared memory with the 3D-RoPE applied on load ("longcat-video-rs"
// section 03-01; section 03-03 for the block list), and keeps an online
// softmax in fp32 registers.  Accuracy path for fp32 inputs; the bf16 path is
// the tcgen05 kernel in attn_sm100.cu.
#include <math.h>

#include "lc_internal.cuh"

namespace {

struct F32Args {
  const float *q, *k, *v, *cond_k, *cond_v;
  float *out, *lse;
  const int *row_ptr, *col_idx;
  int *status;     // device status word (plan checks)
  long long nnz;   // CSR entries
  int n_blocks;    // blocks of the pattern
  const float *tab;
  int T, H, W;
  lc_divmod div_hw, div_w;
  int Nc, Nn, Cb, heads;
  int q_block0;    // first CSR row processed (Cb when only noisy queries)
  int split_kv;    // condition K/V in cond_k / cond_v, noisy K/V in k / v
  int q_mode;      // rows of q / out: 0 all tokens, 1 noisy tokens, 2 condition tokens
  int cond_k_rot;  // cond_k already holds R(k)
  const float *q_nw, *k_nw;  // RMSNorm weights [64] ahead of the rotation, or NULL
  float norm_eps;
  float scale;
};

__device__ __forceinline__ void rope_row(float *x, int n, const F32Args &a, const float *nw) {
  if (nw) {  // RMSNorm first, summed in the library's fixed order
    float c8[8];
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) c8[ch] = lc_sumsq8(x + 8 * ch);
    const float inv = lc_rms_inv(lc_sumsq_tree8(c8), a.norm_eps);
#pragma unroll
    for (int d = 0; d < LC_HEAD_DIM; ++d) x[d] = lc_rms_apply(x[d], inv, __ldg(nw + d));
  }
  int t = lc_div(n, a.div_hw);
  int rem = n - t * a.div_hw.d;
  int h = lc_div(rem, a.div_w);
  int w = rem - h * a.div_w.d;
  const float *cT = a.tab, *sT = cT + a.T * 8;
  const float *cH = sT + a.T * 8, *sH = cH + a.H * 12;
  const float *cW = sH + a.H * 12, *sW = cW + a.W * 12;
#pragma unroll
  for (int p = 0; p < 32; ++p) {
    float c, s;
    if (p < 8) { c = cT[t * 8 + p]; s = sT[t * 8 + p]; }
    else if (p < 20) { c = cH[h * 12 + p - 8]; s = sH[h * 12 + p - 8]; }
    else { c = cW[w * 12 + p - 20]; s = sW[w * 12 + p - 20]; }
    lc_rot_pair(x[2 * p], x[2 * p + 1], c, s, x[2 * p], x[2 * p + 1]);
  }
}

// Address of head `h` of sequence token m (full-sequence index) for K or V.
__device__ __forceinline__ const float *kv_row(const float *full, const float *cond, int b, int m,
                                               int h, const F32Args &a) {
  if (!a.split_kv) {
    long long N = (long long)a.Nc + a.Nn;
    return full + (((long long)b * N + m) * a.heads + h) * LC_HEAD_DIM;
  }
  if (m < a.Nc) return cond + (((long long)b * a.Nc + m) * a.heads + h) * LC_HEAD_DIM;
  return full + (((long long)b * a.Nn + (m - a.Nc)) * a.heads + h) * LC_HEAD_DIM;
}

__global__ void __launch_bounds__(64) attn_f32_kernel(F32Args a) {
  __shared__ float sK[64][LC_HEAD_DIM + 1];
  __shared__ float sV[64][LC_HEAD_DIM + 1];
  const int r = a.q_block0 + blockIdx.x;  // CSR row = query block id
  const int h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
  // Query tokens of block r (full-sequence indices).
  int q_lo, q_hi;
  if (r < a.Cb) { q_lo = 64 * r; q_hi = min(a.Nc, q_lo + 64); }
  else { q_lo = a.Nc + 64 * (r - a.Cb); q_hi = min(a.Nc + a.Nn, q_lo + 64); }
  const int n = q_lo + tid;
  const bool valid = n < q_hi;
  // Row of the q / out tensors that holds token n.
  const int q_row = a.q_mode == 1 ? n - a.Nc : n;
  const long long Nq = a.q_mode == 1 ? a.Nn : (a.q_mode == 2 ? a.Nc : (long long)a.Nc + a.Nn);

  float q[LC_HEAD_DIM], o[LC_HEAD_DIM];
  if (valid) {
    const float *src = a.q + (((long long)b * Nq + q_row) * a.heads + h) * LC_HEAD_DIM;
#pragma unroll
    for (int d = 0; d < LC_HEAD_DIM; ++d) q[d] = src[d];
    rope_row(q, n, a, a.q_nw);
  } else {
#pragma unroll
    for (int d = 0; d < LC_HEAD_DIM; ++d) q[d] = 0.f;
  }
#pragma unroll
  for (int d = 0; d < LC_HEAD_DIM; ++d) {
    q[d] *= a.scale;
    o[d] = 0.f;
  }
  float m_run = -INFINITY, l_run = 0.f;

  int e_lo, e_hi;
  lc_checked_row(a.row_ptr, r, a.nnz, a.status, e_lo, e_hi);
  for (int e = e_lo; e < e_hi; ++e) {
    const int c = a.col_idx[e];
    if (!lc_checked_block(c, a.n_blocks, a.status)) continue;
    int k_lo, k_hi;
    if (c < a.Cb) { k_lo = 64 * c; k_hi = min(a.Nc, k_lo + 64); }
    else { k_lo = a.Nc + 64 * (c - a.Cb); k_hi = min(a.Nc + a.Nn, k_lo + 64); }
    const int kn = k_hi - k_lo;
    __syncthreads();
    if (tid < kn) {
      const int m = k_lo + tid;
      float kr[LC_HEAD_DIM];
      const float *ks = kv_row(a.k, a.cond_k, b, m, h, a);
      const float *vs = kv_row(a.v, a.cond_v, b, m, h, a);
#pragma unroll
      for (int d = 0; d < LC_HEAD_DIM; ++d) kr[d] = ks[d];
      if (!(a.cond_k_rot && m < a.Nc)) rope_row(kr, m, a, a.k_nw);
#pragma unroll
      for (int d = 0; d < LC_HEAD_DIM; ++d) {
        sK[tid][d] = kr[d];
        sV[tid][d] = vs[d];
      }
    }
    __syncthreads();
    for (int j = 0; j < kn; ++j) {
      float s = 0.f;
#pragma unroll
      for (int d = 0; d < LC_HEAD_DIM; ++d) s = fmaf(q[d], sK[j][d], s);
      if (s > m_run) {
        float corr = expf(m_run - s);  // 0 on the first key
        l_run = l_run * corr + 1.f;
#pragma unroll
        for (int d = 0; d < LC_HEAD_DIM; ++d) o[d] = fmaf(o[d], corr, sV[j][d]);
        m_run = s;
      } else {
        float p = expf(s - m_run);
        l_run += p;
#pragma unroll
        for (int d = 0; d < LC_HEAD_DIM; ++d) o[d] = fmaf(p, sV[j][d], o[d]);
      }
    }
  }
  if (!valid) return;
  const float inv = 1.f / l_run;
  float *dst = a.out + (((long long)b * Nq + q_row) * a.heads + h) * LC_HEAD_DIM;
#pragma unroll
  for (int d = 0; d < LC_HEAD_DIM; ++d) dst[d] = o[d] * inv;
  if (a.lse) a.lse[((long long)b * a.heads + h) * Nq + q_row] = m_run + logf(l_run);
}

}  // namespace

lc_status lc_launch_forward_f32(const float *q, const float *k, const float *v,
                                const float *cond_k, const float *cond_v, float *out, float *lse,
                                int batch, int heads, float scale, lc_fwd_mode mode,
                                bool cond_k_rotated, const lc_qk_norm &norm,
                                const lc_bsa_plan_s *plan, const lc_rope3d_s *rope,
                                int *dev_status, cudaStream_t stream) {
  F32Args a;
  a.q = q; a.k = k; a.v = v; a.cond_k = cond_k; a.cond_v = cond_v;
  a.out = out; a.lse = lse;
  a.row_ptr = plan->row_ptr; a.col_idx = plan->col_idx;
  a.status = dev_status;
  a.nnz = plan->nnz;
  a.n_blocks = plan->Cb + plan->Nb;
  a.tab = rope->tab;
  a.T = rope->T; a.H = rope->H; a.W = rope->W;
  a.div_hw = lc_make_divmod(rope->H * rope->W);
  a.div_w = lc_make_divmod(rope->W);
  a.Nc = plan->Nc; a.Nn = plan->Nn; a.Cb = plan->Cb; a.heads = heads;
  a.split_kv = mode != LC_FWD_FULL;
  a.q_mode = mode == LC_FWD_CACHED ? 1 : (mode == LC_FWD_COND ? 2 : 0);
  a.cond_k_rot = (mode != LC_FWD_FULL && cond_k_rotated) ? 1 : 0;
  a.q_block0 = mode == LC_FWD_CACHED ? plan->Cb : 0;
  a.scale = scale;
  a.q_nw = norm.q_w;
  a.k_nw = norm.k_w;
  a.norm_eps = norm.eps;
  int nrows = mode == LC_FWD_CACHED ? plan->Nb : (mode == LC_FWD_COND ? plan->Cb : plan->nq);
  if (nrows == 0) return LC_OK;
  LC_CUDA_TRY(cudaStreamWaitEvent(stream, plan->ready, 0));
  LC_CUDA_TRY(cudaStreamWaitEvent(stream, rope->ready, 0));
  dim3 grid(nrows, heads, batch);
  attn_f32_kernel<<<grid, 64, 0, stream>>>(a);
  LC_CUDA_TRY(cudaGetLastError());
  return LC_OK;
}
