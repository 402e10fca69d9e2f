// ring.cu -- device pieces of ring context parallelism: the sequence is cut
// into contiguous shards, each rank keeps its queries and passes the K/V
// shards around a ring, and the partial results over the K/V shards are
// combined by their log-sum-exp (myzaker / QbitAI "背后技术原理": block-sparse
// attention combined with context-parallel ring block-sparse attention).
//
//   shard_fill   rows of a shard plan's query range that no key of the K/V
//                shard reaches as a group (no plan entries): out = 0,
//                lse = -inf, so every row of a shard result is defined.
//   lse_merge    (o, lse) <- merge((o, lse), (o_p, lse_p)): with
//                m = max(lse, lse_p), w = e^(lse - m), w_p = e^(lse_p - m):
//                o = (w o + w_p o_p) / (w + w_p), lse = m + log(w + w_p).
//                Both -inf: the row stays (0, -inf).
//   lse_merge_parts  the same over P parts at once (one pass: a ring's
//                partial results kept until the last step, then combined).
// All are HBM-bound elementwise passes; eight lanes per (batch, token, head)
// row, each on 8 channels with 16- / 32-byte vector accesses.
#include <cuda_bf16.h>
#include <math.h>

#include "lc_internal.cuh"
#include "lc_vec8.cuh"

namespace {

using lcvec::ld8;
using lcvec::st8;

struct FillArgs {
  const int *grp_ptr;
  int G, gc, Cb, Nc, Nn;
  int qlo, qhi;         // the plan's query blocks
  long long q_lo, q_n;  // its query tokens
  int batch, heads;
};

// Grid (group, slice): each CTA clears one of gridDim.y slices of a group's
// rows; groups outside the query range or with entries return at once.
template <typename T>
__global__ void shard_fill_kernel(FillArgs a, T *out, float *lse) {
  const int g = blockIdx.x;
  const int first = g < a.gc ? 4 * g : a.Cb + 4 * (g - a.gc);
  if (first < a.qlo || first >= a.qhi) return;
  if (a.grp_ptr[g + 1] != a.grp_ptr[g]) return;
  const long long seg_end = g < a.gc ? a.Nc : (long long)a.Nc + a.Nn;
  const long long t0 = g < a.gc ? 256LL * g : a.Nc + 256LL * (g - a.gc);
  const long long t1 = t0 + 256 < seg_end ? t0 + 256 : seg_end;
  long long r0 = t0 - a.q_lo, r1 = t1 - a.q_lo;  // rows of the shard buffers
  r0 = r0 < 0 ? 0 : r0;
  r1 = r1 > a.q_n ? a.q_n : r1;
  // this CTA's slice of the rows
  const long long nr = r1 - r0, per = (nr + gridDim.y - 1) / gridDim.y;
  const long long s0 = r0 + per * blockIdx.y;
  const long long s1 = s0 + per < r1 ? s0 + per : r1;
  if (s0 >= s1) return;
  // out[b, s0:s1] is one contiguous span per batch entry (whole rows: a
  // multiple of 16 bytes).
  const long long vec = (s1 - s0) * a.heads * LC_HEAD_DIM * (long long)sizeof(T) / 16;
  const long long nl = (s1 - s0) * a.heads;
  for (int b = 0; b < a.batch; ++b) {
    uint4 *dst = reinterpret_cast<uint4 *>(out + ((long long)b * a.q_n + s0) * a.heads * LC_HEAD_DIM);
    for (long long i = threadIdx.x; i < vec; i += blockDim.x) dst[i] = make_uint4(0, 0, 0, 0);
    for (long long i = threadIdx.x; i < nl; i += blockDim.x) {
      const int h = (int)(i / (s1 - s0));
      const long long r = s0 + i % (s1 - s0);
      lse[((long long)b * a.heads + h) * a.q_n + r] = -INFINITY;
    }
  }
}

template <typename T>
__global__ void lse_merge_kernel(float *o_acc, float *lse_acc, const T *o_part,
                                 const float *lse_part, T *out, long long rows, long long n,
                                 int heads, int init) {
  const long long gid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  const long long i = gid >> 3;  // (b * n + t) * heads + h
  const int ch = (int)(gid & 7);
  if (i >= rows) return;
  const int h = (int)(i % heads);
  const long long bt = i / heads;
  const long long b = bt / n, t = bt - b * n;
  const long long li = (b * heads + h) * n + t;
  const long long oi = i * LC_HEAD_DIM + 8 * ch;
  float p[8], o[8];
  ld8(o_part + oi, p);
  const float lp = lse_part[li];
  float l;
  if (init) {
    l = lp;
#pragma unroll
    for (int e = 0; e < 8; ++e) o[e] = lp == -INFINITY ? 0.f : p[e];
  } else {
    ld8(o_acc + oi, o);
    const float la = lse_acc[li];
    const float m = fmaxf(la, lp);
    if (m == -INFINITY) {
      l = -INFINITY;
#pragma unroll
      for (int e = 0; e < 8; ++e) o[e] = 0.f;
    } else {
      const float wa = expf(la - m), wp = expf(lp - m);  // one of them is 1
      const float inv = 1.f / (wa + wp);
      const float ca = wa * inv, cp = wp * inv;
#pragma unroll
      for (int e = 0; e < 8; ++e)
        o[e] = (wa > 0.f ? ca * o[e] : 0.f) + (wp > 0.f ? cp * p[e] : 0.f);
      l = m + logf(wa + wp);
    }
  }
  if (out)
    st8(out + oi, o);
  else
    st8(o_acc + oi, o);
  if (ch == 0) lse_acc[li] = l;
}

// P partial results of the same rows over disjoint key sets -> the result
// over all of them: m = max_i lse_i, w_i = e^(lse_i - m),
// o = sum_i w_i o_i / sum_i w_i, lse = m + log sum_i w_i (all -inf: 0, -inf).
// One pass over the parts' outputs (a part of weight 0 is not added).
template <typename T>
__global__ void lse_merge_parts_kernel(const T *parts, const float *lses, int n_parts, T *out,
                                       float *lse_out, long long rows, long long n, int heads) {
  const long long gid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  const long long i = gid >> 3;  // (b * n + t) * heads + h
  const int ch = (int)(gid & 7);
  if (i >= rows) return;
  const int h = (int)(i % heads);
  const long long bt = i / heads;
  const long long b = bt / n, t = bt - b * n;
  const long long li = (b * heads + h) * n + t;
  const long long oi = i * LC_HEAD_DIM + 8 * ch;
  const long long o_stride = rows * LC_HEAD_DIM, l_stride = rows;  // per part
  float m = -INFINITY;
  for (int k = 0; k < n_parts; ++k) m = fmaxf(m, lses[k * l_stride + li]);
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float wsum = 0.f;
  if (m != -INFINITY) {
    // four parts at a time, their loads issued together; a part of weight 0
    // is read but not added (its values may be anything)
    int k = 0;
    for (; k + 4 <= n_parts; k += 4) {
      float w[4], v[4][8];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        w[u] = expf(lses[(k + u) * l_stride + li] - m);
        ld8(parts + (k + u) * o_stride + oi, v[u]);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (w[u] > 0.f) {
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[e] = fmaf(w[u], v[u][e], acc[e]);
          wsum += w[u];
        }
      }
    }
    for (; k < n_parts; ++k) {
      const float w = expf(lses[k * l_stride + li] - m);
      if (w > 0.f) {
        float v[8];
        ld8(parts + k * o_stride + oi, v);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = fmaf(w, v[e], acc[e]);
        wsum += w;
      }
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] *= inv;
  st8(out + oi, acc);
  if (ch == 0 && lse_out) lse_out[li] = m == -INFINITY ? -INFINITY : m + logf(wsum);
}

}  // namespace

lc_status lc_launch_shard_fill(const lc_bsa_plan_s *plan, void *out, float *lse, int batch,
                               int heads, lc_dtype dtype, cudaStream_t stream) {
  if (!plan->fill_needed) return LC_OK;  // every group of the query range has entries
  FillArgs a;
  a.grp_ptr = plan->grp_ptr;
  a.G = plan->G; a.gc = plan->gc; a.Cb = plan->Cb; a.Nc = plan->Nc; a.Nn = plan->Nn;
  a.qlo = plan->qlo; a.qhi = plan->qhi;
  a.q_lo = lc_block_token(plan, plan->qlo);
  a.q_n = lc_block_token(plan, plan->qhi) - a.q_lo;
  a.batch = batch; a.heads = heads;
  if (a.q_n <= 0) return LC_OK;
  LC_CUDA_TRY(cudaStreamWaitEvent(stream, plan->ready, 0));
  const dim3 grid(plan->G, 16);  // 16 slices of up to 16 rows per group
  if (dtype == LC_DTYPE_F32)
    shard_fill_kernel<float><<<grid, 256, 0, stream>>>(a, static_cast<float *>(out), lse);
  else
    shard_fill_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(
        a, static_cast<__nv_bfloat16 *>(out), lse);
  LC_CUDA_TRY(cudaGetLastError());
  return LC_OK;
}

lc_status lc_launch_lse_merge(float *o_acc, float *lse_acc, const void *o_part,
                              const float *lse_part, void *out, int batch, long long n, int heads,
                              lc_dtype dtype, bool init, cudaStream_t stream) {
  const long long rows = (long long)batch * n * heads;
  if (rows == 0) return LC_OK;
  const long long threads = rows * 8;
  const long long blocks = (threads + 255) / 256;
  if (blocks > 0x7FFFFFFFLL) return LC_ERR_UNSUPPORTED;  // past the grid's x limit
  const unsigned grid = (unsigned)blocks;
  if (dtype == LC_DTYPE_F32)
    lse_merge_kernel<float><<<grid, 256, 0, stream>>>(o_acc, lse_acc,
                                                      static_cast<const float *>(o_part), lse_part,
                                                      static_cast<float *>(out), rows, n, heads,
                                                      init ? 1 : 0);
  else
    lse_merge_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(
        o_acc, lse_acc, static_cast<const __nv_bfloat16 *>(o_part), lse_part,
        static_cast<__nv_bfloat16 *>(out), rows, n, heads, init ? 1 : 0);
  LC_CUDA_TRY(cudaGetLastError());
  return LC_OK;
}

lc_status lc_launch_lse_merge_parts(const void *parts, const float *lses, int n_parts, void *out,
                                    float *lse_out, int batch, long long n, int heads,
                                    lc_dtype dtype, cudaStream_t stream) {
  const long long rows = (long long)batch * n * heads;
  if (rows == 0) return LC_OK;
  const long long blocks = (rows * 8 + 255) / 256;
  if (blocks > 0x7FFFFFFFLL) return LC_ERR_UNSUPPORTED;  // past the grid's x limit
  const unsigned grid = (unsigned)blocks;
  if (dtype == LC_DTYPE_F32)
    lse_merge_parts_kernel<float><<<grid, 256, 0, stream>>>(
        static_cast<const float *>(parts), lses, n_parts, static_cast<float *>(out), lse_out,
        rows, n, heads);
  else
    lse_merge_parts_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(parts), lses, n_parts,
        static_cast<__nv_bfloat16 *>(out), lse_out, rows, n, heads);
  LC_CUDA_TRY(cudaGetLastError());
  return LC_OK;
}
