// rope.cu -- partitioned 3D-RoPE tables and the standalone rotation kernel.
//
// "longcat-video-rs" header card ("16T + 24H + 24W ... norm-conserving
// spatiotemporal rotary pairs") and section 03-01: a 64-D head is split into
// a temporal slice (channels [0,16)), a height slice ([16,40)) and a width
// slice ([40,64)); pair (c, c+1) of a slice of width d, pair index k, turns by
// pos * theta^(-2k/d) with pos the token's t, h or w.
#include <math.h>

#include <new>

#include "lc_internal.cuh"
#include "lc_vec8.cuh"
#include <cuda_bf16.h>

namespace {

// One thread per table entry; angles and cos/sin in fp64, stored fp32.
__global__ void rope_tables_kernel(float *tab, int T, int H, int W, double theta, int dt, int dh,
                                   int dw) {
  long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  const int npos[3] = {T, H, W};
  const int dims[3] = {dt, dh, dw};
  long long base = 0;
  for (int a = 0; a < 3; ++a) {
    long long half = (long long)npos[a] * (dims[a] / 2);
    if (i < base + 2 * half) {
      long long j = i - base;
      bool is_sin = j >= half;
      if (is_sin) j -= half;
      int pos = (int)(j / (dims[a] / 2));
      int k = (int)(j % (dims[a] / 2));
      double omega = pow(theta, -2.0 * (double)k / (double)dims[a]);
      double phi = (double)pos * omega;
      tab[i] = (float)(is_sin ? sin(phi) : cos(phi));
      return;
    }
    base += 2 * half;
  }
}

// Rotate the 4 channel pairs of 8-channel chunk `ch` (0..7) of a 64-D head.
__device__ __forceinline__ void rotate_chunk(float (&x)[8], int ch, int t, int h, int w,
                                             const float *tab, int T, int H, int W) {
  const float *c, *s;
  if (ch < 2) {
    c = tab + t * 8 + 4 * ch;
    s = c + T * 8;
  } else if (ch < 5) {
    c = tab + T * 16 + h * 12 + 4 * (ch - 2);
    s = c + H * 12;
  } else {
    c = tab + T * 16 + H * 24 + w * 12 + 4 * (ch - 5);
    s = c + W * 12;
  }
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const float a = x[2 * p], b = x[2 * p + 1];
    lc_rot_pair(a, b, c[p], s[p], x[2 * p], x[2 * p + 1]);
  }
}

template <typename Tin>
__global__ void rope_apply_kernel(const Tin *x, Tin *out, long long n_chunks, int heads,
                                  long long ntok, long long tok_offset, const float *tab, int T,
                                  int H, int W, lc_divmod div_hw, lc_divmod div_w,
                                  const float *nw, float eps) {
  const unsigned group = 0xFFu << (threadIdx.x & 24);  // the 8 lanes holding one row
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n_chunks;
       i += (long long)gridDim.x * blockDim.x) {
    int ch = (int)(i & 7);
    long long tokhead = i >> 3;
    long long tok = (tokhead / heads) % ntok;
    int n = (int)(tok + tok_offset);
    int t = lc_div(n, div_hw);
    int rem = n - t * div_hw.d;
    int h = lc_div(rem, div_w);
    int w = rem - h * div_w.d;
    float v[8];
    lcvec::ld8(x + i * 8, v);  // one 16- / 32-byte load (x is 16-byte aligned)
    if (nw) {  // uniform: every lane of a group is in the loop together
      const float inv = lc_rms_inv(lc_sumsq_lanes8(lc_sumsq8(v), group), eps);
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = lc_rms_apply(v[e], inv, __ldg(nw + 8 * ch + e));
    }
    rotate_chunk(v, ch, t, h, w, tab, T, H, W);
    lcvec::st8(out + i * 8, v);
  }
}

}  // namespace

extern "C" lc_status lc_rope3d_tables(lc_rope3d *out, int T, int H, int W, double theta, int dim_t,
                                      int dim_h, int dim_w, void *stream) {
  if (!out || T <= 0 || H <= 0 || W <= 0 || !(theta > 0.0) || dim_t <= 0 || dim_h <= 0 ||
      dim_w <= 0 || (dim_t & 1) || (dim_h & 1) || (dim_w & 1))
    return LC_ERR_INVALID_ARGUMENT;
  if (dim_t != 16 || dim_h != 24 || dim_w != 24) return LC_ERR_UNSUPPORTED;
  if ((long long)T * H * W >= (1LL << 24) || (long long)H * W >= (1LL << 16))
    return LC_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  lc_rope3d_s *r = new (std::nothrow) lc_rope3d_s();
  if (!r) return LC_ERR_OUT_OF_MEMORY;
  r->T = T; r->H = H; r->W = W; r->theta = theta;
  r->dt = dim_t; r->dh = dim_h; r->dw = dim_w;
  r->n_floats = (long long)T * dim_t + (long long)H * dim_h + (long long)W * dim_w;
  lc_status s = lc_from_cuda(cudaGetDevice(&r->device));
  if (s != LC_OK) { delete r; return s; }
  cudaError_t e = cudaMallocAsync(&r->tab, sizeof(float) * r->n_floats, st);
  if (e != cudaSuccess) { delete r; return lc_from_cuda(e); }
  int tpb = 256;
  int nb = (int)((r->n_floats + tpb - 1) / tpb);
  rope_tables_kernel<<<nb, tpb, 0, st>>>(r->tab, T, H, W, theta, dim_t, dim_h, dim_w);
  e = cudaGetLastError();
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&r->ready, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventRecord(r->ready, st);
  if (e != cudaSuccess) {
    cudaFreeAsync(r->tab, st);
    delete r;
    return lc_from_cuda(e);
  }
  *out = r;
  return LC_OK;
}

extern "C" lc_status lc_rope3d_destroy(lc_rope3d rope, void *stream) {
  if (!rope) return LC_OK;
  cudaError_t e = cudaFreeAsync(rope->tab, static_cast<cudaStream_t>(stream));
  cudaEventDestroy(rope->ready);
  delete rope;
  return lc_from_cuda(e);
}

extern "C" lc_status lc_rope3d_copy_tables(lc_rope3d rope, float *host, void *stream) {
  if (!rope || !host) return LC_ERR_INVALID_ARGUMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  LC_CUDA_TRY(cudaStreamWaitEvent(st, rope->ready, 0));
  LC_CUDA_TRY(cudaMemcpyAsync(host, rope->tab, sizeof(float) * rope->n_floats,
                              cudaMemcpyDeviceToHost, st));
  LC_CUDA_TRY(cudaStreamSynchronize(st));
  return LC_OK;
}

lc_status lc_rotate_rows(const void *x, void *out, int batch, long long ntok, int heads,
                         long long tok_offset, lc_dtype dtype, const lc_rope3d_s *rope,
                         const float *norm_w, float eps, cudaStream_t st) {
  long long n_chunks = (long long)batch * ntok * heads * (LC_HEAD_DIM / 8);
  if (n_chunks == 0) return LC_OK;
  int tpb = 256;
  long long want = (n_chunks + tpb - 1) / tpb;
  int nb = (int)(want < 148LL * 16 ? want : 148LL * 16);
  lc_divmod dhw = lc_make_divmod(rope->H * rope->W), dw = lc_make_divmod(rope->W);
  LC_CUDA_TRY(cudaStreamWaitEvent(st, rope->ready, 0));
  if (dtype == LC_DTYPE_F32)
    rope_apply_kernel<float><<<nb, tpb, 0, st>>>(static_cast<const float *>(x),
                                                 static_cast<float *>(out), n_chunks, heads, ntok,
                                                 tok_offset, rope->tab, rope->T, rope->H, rope->W,
                                                 dhw, dw, norm_w, eps);
  else
    rope_apply_kernel<__nv_bfloat16><<<nb, tpb, 0, st>>>(
        static_cast<const __nv_bfloat16 *>(x), static_cast<__nv_bfloat16 *>(out), n_chunks,
        heads, ntok, tok_offset, rope->tab, rope->T, rope->H, rope->W, dhw, dw, norm_w, eps);
  LC_CUDA_TRY(cudaGetLastError());
  return LC_OK;
}

extern "C" lc_status lc_rope3d_apply_ex(const void *x, void *out, int batch, long long ntok,
                                        int heads, int head_dim, long long tok_offset,
                                        lc_dtype dtype, const float *norm_weight, float norm_eps,
                                        lc_rope3d rope, void *stream) {
  if (!x || !out || !rope || batch <= 0 || ntok <= 0 || heads <= 0 || tok_offset < 0)
    return LC_ERR_INVALID_ARGUMENT;
  if (dtype != LC_DTYPE_BF16 && dtype != LC_DTYPE_F32) return LC_ERR_INVALID_ARGUMENT;
  if (head_dim != LC_HEAD_DIM) return LC_ERR_UNSUPPORTED;
  if (tok_offset + ntok > (long long)rope->T * rope->H * rope->W) return LC_ERR_INVALID_ARGUMENT;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(out)) & 15)
    return LC_ERR_INVALID_ARGUMENT;
  if (norm_weight && ((reinterpret_cast<uintptr_t>(norm_weight) & 3) ||
                      !(norm_eps >= 0.f && norm_eps <= 3.0e38f)))
    return LC_ERR_INVALID_ARGUMENT;
  int dev = -1;
  LC_CUDA_TRY(cudaGetDevice(&dev));
  if (dev != rope->device) return LC_ERR_INVALID_ARGUMENT;
  return lc_rotate_rows(x, out, batch, ntok, heads, tok_offset, dtype, rope, norm_weight,
                        norm_weight ? norm_eps : 0.f, static_cast<cudaStream_t>(stream));
}

extern "C" lc_status lc_rope3d_apply(const void *x, void *out, int batch, long long ntok, int heads,
                                     int head_dim, long long tok_offset, lc_dtype dtype,
                                     lc_rope3d rope, void *stream) {
  if (!x || !out || !rope || batch <= 0 || ntok <= 0 || heads <= 0 || tok_offset < 0)
    return LC_ERR_INVALID_ARGUMENT;
  if (dtype != LC_DTYPE_BF16 && dtype != LC_DTYPE_F32) return LC_ERR_INVALID_ARGUMENT;
  if (head_dim != LC_HEAD_DIM) return LC_ERR_UNSUPPORTED;
  if (tok_offset + ntok > (long long)rope->T * rope->H * rope->W) return LC_ERR_INVALID_ARGUMENT;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(out)) & 15)
    return LC_ERR_INVALID_ARGUMENT;
  int dev = -1;
  LC_CUDA_TRY(cudaGetDevice(&dev));
  if (dev != rope->device) return LC_ERR_INVALID_ARGUMENT;
  return lc_rotate_rows(x, out, batch, ntok, heads, tok_offset, dtype, rope, nullptr, 0.f,
                        static_cast<cudaStream_t>(stream));
}
