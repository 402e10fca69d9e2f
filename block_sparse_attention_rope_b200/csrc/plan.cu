// plan.cu -- device-side planner of the block-sparse pattern.
//
// Pattern ("longcat-video-rs", section 03-03 "Block-Sparse & Multi-Audio" and
// the section 02 table row "block=64, local=2, stride=4"; myzaker / QbitAI,
// "背后技术原理" for the condition frames):
//   condition query block r < Cb  -> every condition key block;
//   noisy query block Cb+i        -> every condition key block, plus noisy key
//                                    block Cb+j iff |i-j| <= local or
//                                    (stride > 0 and j % stride == 0).
//
// Kernels (all tiny, run once per shape):
//   row_scan    one warp per query block: count its key blocks by ballot and
//               the attended token pairs;
//   group_count one warp per group of 4 query blocks: size of the union list;
//   scan        one CTA: exclusive scans -> row_ptr, grp_ptr; checks nnz;
//   row_fill    one warp per query block: ascending key ids -> col_idx;
//   group_fill  one warp per group: union entries (key id | member mask << 24);
//   order       one thread per group: rank by entry count, longest first;
//   col_scan,   one warp per key block: the transpose (CSC), ascending query
//   col_fill    block ids attending it (walked by the backward pass).
#include <algorithm>
#include <new>

#include "lc_internal.cuh"

namespace {

struct PlanGeom {
  int Nc, Nn, Cb, Nb, nq, gc, gn, G, local, stride;
  int kgc, kgn, KG;  // key groups of 2 blocks (backward)
  int qlo, qhi, klo, khi;  // the plan covers query blocks [qlo, qhi) x key blocks [klo, khi)
};

// The pattern (query block r attends key block c), restricted to the plan's
// block ranges.  Same rule on the host (sizing) and the device.
__host__ __device__ __forceinline__ bool attends(int r, int c, const PlanGeom &g) {
  if (r < g.qlo || r >= g.qhi || c < g.klo || c >= g.khi) return false;
  if (r < g.Cb) return c < g.Cb;
  if (c < g.Cb) return true;
  int i = r - g.Cb, j = c - g.Cb;
  int d = i > j ? i - j : j - i;
  return d <= g.local || (g.stride > 0 && (j % g.stride) == 0);
}

__device__ __forceinline__ int block_tokens(int b, const PlanGeom &g) {
  if (b < g.Cb) return min(LC_BLOCK, g.Nc - LC_BLOCK * b);
  return min(LC_BLOCK, g.Nn - LC_BLOCK * (b - g.Cb));
}

// Group gi covers query blocks first..first+cnt-1 (global block ids).
__device__ __forceinline__ void group_members(int gi, const PlanGeom &g, int *first, int *cnt) {
  if (gi < g.gc) {
    *first = 4 * gi;
    *cnt = min(4, g.Cb - 4 * gi);
  } else {
    *first = g.Cb + 4 * (gi - g.gc);
    *cnt = min(4, g.Nb - 4 * (gi - g.gc));
  }
}

// Key group ki: up to two key blocks (global block ids) of one segment whose
// query lists are alike, so that the backward pass computes few masked
// pairs.  Condition blocks pair in order (all are attended by every query
// block).  In the noisy segment with strided globals, the global blocks
// (j % stride == 0, attended by every noisy query block) pair with each
// other, and the local-only blocks pair in order; otherwise blocks pair in
// order.
__device__ __forceinline__ void kgroup_members(int ki, const PlanGeom &g, int *blk, int *cnt) {
  if (ki < g.kgc) {
    blk[0] = 2 * ki;
    *cnt = min(2, g.Cb - 2 * ki);
    blk[1] = blk[0] + 1;
    return;
  }
  const int gi = ki - g.kgc;
  if (g.stride <= 1) {
    blk[0] = g.Cb + 2 * gi;
    *cnt = min(2, g.Nb - 2 * gi);
    blk[1] = blk[0] + 1;
    return;
  }
  const int s = g.stride;
  const int n_glob = (g.Nb + s - 1) / s;
  const int kg_glob = (n_glob + 1) / 2;
  if (gi < kg_glob) {
    blk[0] = g.Cb + (2 * gi) * s;
    *cnt = min(2, n_glob - 2 * gi);
    blk[1] = g.Cb + (2 * gi + 1) * s;
  } else {
    const int li = 2 * (gi - kg_glob);  // index among the non-multiples of s
    const int n_loc = g.Nb - n_glob;
    *cnt = min(2, n_loc - li);
    blk[0] = g.Cb + (li / (s - 1)) * s + li % (s - 1) + 1;
    blk[1] = g.Cb + ((li + 1) / (s - 1)) * s + (li + 1) % (s - 1) + 1;
  }
}

// Key blocks of every key group, for the backward kernel: (first, second or -1).
__global__ void kgroup_blocks_kernel(PlanGeom g, int2 *kg_blk) {
  const int ki = blockIdx.x * blockDim.x + threadIdx.x;
  if (ki >= g.KG) return;
  int blk[2], cnt;
  kgroup_members(ki, g, blk, &cnt);
  kg_blk[ki] = make_int2(blk[0], cnt > 1 ? blk[1] : -1);
}

// One warp per key group: size of the union of its members' query lists.
__global__ void kgroup_count_kernel(PlanGeom g, int *cnt_out) {
  int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  int lane = threadIdx.x & 31;
  if (warp >= g.KG) return;
  int blk[2], cnt;
  kgroup_members(warp, g, blk, &cnt);
  int n = 0;
  for (int r0 = 0; r0 < g.nq; r0 += 32) {
    int r = r0 + lane;
    bool any = false;
    if (r < g.nq)
      for (int m = 0; m < cnt; ++m) any |= attends(r, blk[m], g);
    n += __popc(__ballot_sync(0xffffffffu, any));
  }
  if (lane == 0) cnt_out[warp] = n;
}

// One warp per key group: union entries (query block id | member mask << 24).
__global__ void kgroup_fill_kernel(PlanGeom g, const int *ptr, uint32_t *ent, long long cap,
                                   int *err) {
  int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  int lane = threadIdx.x & 31;
  if (warp >= g.KG) return;
  int blk[2], cnt;
  kgroup_members(warp, g, blk, &cnt);
  long long pos = ptr[warp];
  long long end = ptr[warp + 1];
  for (int r0 = 0; r0 < g.nq; r0 += 32) {
    int r = r0 + lane;
    uint32_t mask = 0;
    if (r < g.nq)
      for (int m = 0; m < cnt; ++m) mask |= attends(r, blk[m], g) ? (1u << m) : 0u;
    unsigned bal = __ballot_sync(0xffffffffu, mask != 0);
    if (mask) {
      long long at = pos + __popc(bal & ((1u << lane) - 1u));
      if (at < end && at < cap)
        ent[at] = (uint32_t)r | (mask << 24);
      else
        atomicOr(err, 64);
    }
    pos += __popc(bal);
  }
}

__global__ void row_scan_kernel(PlanGeom g, int *row_cnt, unsigned long long *pairs) {
  int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  int lane = threadIdx.x & 31;
  if (warp >= g.nq) return;
  int r = warp;
  int ncols = g.Cb + g.Nb;
  int cnt = 0;
  unsigned long long keys = 0;
  for (int c0 = 0; c0 < ncols; c0 += 32) {
    int c = c0 + lane;
    bool a = c < ncols && attends(r, c, g);
    cnt += __popc(__ballot_sync(0xffffffffu, a));
    if (a) keys += (unsigned long long)block_tokens(c, g);
  }
  for (int o = 16; o > 0; o >>= 1) keys += __shfl_xor_sync(0xffffffffu, keys, o);
  if (lane == 0) {
    row_cnt[r] = cnt;
    unsigned long long p = keys * (unsigned long long)block_tokens(r, g);
    atomicAdd(&pairs[0], p);
    if (r >= g.Cb) atomicAdd(&pairs[1], p);
  }
}

__global__ void group_count_kernel(PlanGeom g, int *grp_cnt) {
  int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  int lane = threadIdx.x & 31;
  if (warp >= g.G) return;
  int first, cnt;
  group_members(warp, g, &first, &cnt);
  int ncols = g.Cb + g.Nb;
  int n = 0;
  for (int c0 = 0; c0 < ncols; c0 += 32) {
    int c = c0 + lane;
    bool any = false;
    if (c < ncols)
      for (int m = 0; m < cnt; ++m) any |= attends(first + m, c, g);
    n += __popc(__ballot_sync(0xffffffffu, any));
  }
  if (lane == 0) grp_cnt[warp] = n;
}

// Exclusive scan of n ints by one CTA of 1024 threads (chunked).
__device__ void block_exclusive_scan(const int *in, int *out, int n, long long *total) {
  __shared__ long long warp_sums[32];
  __shared__ long long carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < n; base += blockDim.x) {
    int i = base + threadIdx.x;
    long long v = i < n ? in[i] : 0;
    long long x = v;
    int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    for (int o = 1; o < 32; o <<= 1) {
      long long y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[w] = x;
    __syncthreads();
    if (w == 0) {
      long long s = lane < (int)(blockDim.x >> 5) ? warp_sums[lane] : 0;
      for (int o = 1; o < 32; o <<= 1) {
        long long y = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += y;
      }
      warp_sums[lane] = s;  // inclusive sums of warps
    }
    __syncthreads();
    long long before = carry + (w > 0 ? warp_sums[w - 1] : 0) + x - v;
    if (i < n) out[i] = (int)before;
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry = before + v;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    out[n] = (int)carry;
    *total = carry;
  }
}

__global__ void scan_kernel(PlanGeom g, const int *row_cnt, int *row_ptr, const int *grp_cnt,
                            int *grp_ptr, const int *col_cnt, int *col_ptr, const int *kgrp_cnt,
                            int *kgrp_ptr, long long nnz_expect, int *err) {
  __shared__ long long tot;
  block_exclusive_scan(row_cnt, row_ptr, g.nq, &tot);
  __syncthreads();
  if (threadIdx.x == 0 && tot != nnz_expect) atomicOr(err, 1);
  __syncthreads();
  block_exclusive_scan(grp_cnt, grp_ptr, g.G, &tot);
  __syncthreads();
  if (threadIdx.x == 0 && tot > nnz_expect) atomicOr(err, 2);
  __syncthreads();
  block_exclusive_scan(col_cnt, col_ptr, g.nq, &tot);
  __syncthreads();
  if (threadIdx.x == 0 && tot != nnz_expect) atomicOr(err, 16);
  __syncthreads();
  block_exclusive_scan(kgrp_cnt, kgrp_ptr, g.KG, &tot);
  __syncthreads();
  if (threadIdx.x == 0 && tot > nnz_expect) atomicOr(err, 128);
}

// Transpose of the pattern, one warp per key block c: how many query blocks
// attend it, then their ids in ascending order.
__global__ void col_scan_kernel(PlanGeom g, int *col_cnt) {
  int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  int lane = threadIdx.x & 31;
  if (warp >= g.nq) return;
  int c = warp, cnt = 0;
  for (int r0 = 0; r0 < g.nq; r0 += 32) {
    int r = r0 + lane;
    cnt += __popc(__ballot_sync(0xffffffffu, r < g.nq && attends(r, c, g)));
  }
  if (lane == 0) col_cnt[c] = cnt;
}

__global__ void col_fill_kernel(PlanGeom g, const int *col_ptr, int *row_idx, long long nnz,
                                int *err) {
  int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  int lane = threadIdx.x & 31;
  if (warp >= g.nq) return;
  int c = warp;
  long long pos = col_ptr[c];
  long long end = col_ptr[c + 1];
  for (int r0 = 0; r0 < g.nq; r0 += 32) {
    int r = r0 + lane;
    bool a = r < g.nq && attends(r, c, g);
    unsigned bal = __ballot_sync(0xffffffffu, a);
    if (a) {
      long long at = pos + __popc(bal & ((1u << lane) - 1u));
      if (at < end && at < nnz)
        row_idx[at] = r;
      else
        atomicOr(err, 32);
    }
    pos += __popc(bal);
  }
}

__global__ void row_fill_kernel(PlanGeom g, const int *row_ptr, int *col_idx, long long nnz,
                                int *err) {
  int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  int lane = threadIdx.x & 31;
  if (warp >= g.nq) return;
  int r = warp;
  int ncols = g.Cb + g.Nb;
  long long pos = row_ptr[r];
  long long end = row_ptr[r + 1];
  for (int c0 = 0; c0 < ncols; c0 += 32) {
    int c = c0 + lane;
    bool a = c < ncols && attends(r, c, g);
    unsigned bal = __ballot_sync(0xffffffffu, a);
    if (a) {
      long long at = pos + __popc(bal & ((1u << lane) - 1u));
      if (at < end && at < nnz)
        col_idx[at] = c;
      else
        atomicOr(err, 4);
    }
    pos += __popc(bal);
  }
}

__global__ void group_fill_kernel(PlanGeom g, const int *grp_ptr, uint32_t *ent, long long cap,
                                  int *err) {
  int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  int lane = threadIdx.x & 31;
  if (warp >= g.G) return;
  int first, cnt;
  group_members(warp, g, &first, &cnt);
  int ncols = g.Cb + g.Nb;
  long long pos = grp_ptr[warp];
  long long end = grp_ptr[warp + 1];
  for (int c0 = 0; c0 < ncols; c0 += 32) {
    int c = c0 + lane;
    uint32_t mask = 0;
    if (c < ncols)
      for (int m = 0; m < cnt; ++m) mask |= attends(first + m, c, g) ? (1u << m) : 0u;
    unsigned bal = __ballot_sync(0xffffffffu, mask != 0);
    if (mask) {
      long long at = pos + __popc(bal & ((1u << lane) - 1u));
      if (at < end && at < cap)
        ent[at] = (uint32_t)c | (mask << 24);
      else
        atomicOr(err, 8);
    }
    pos += __popc(bal);
  }
}

__global__ void order_kernel(int n, const int *grp_cnt, int *order) {
  int gi = blockIdx.x * blockDim.x + threadIdx.x;
  if (gi >= n) return;
  int mine = grp_cnt[gi];
  int rank = 0;
  for (int o = 0; o < n; ++o) {
    int c = grp_cnt[o];
    rank += (c > mine) || (c == mine && o < gi);
  }
  order[rank] = gi;
}

// Key blocks of noisy query block i (closed form, for sizing only).
long long noisy_row_count(long long i, long long Nb, long long local, long long stride) {
  long long lo = std::max(0LL, i - local), hi = std::min(Nb - 1, i + local);
  long long L = hi - lo + 1;
  if (stride <= 0) return L;
  long long glob = (Nb + stride - 1) / stride;
  long long in_win = hi / stride - (lo > 0 ? (lo - 1) / stride : -1);
  return L + glob - in_win;
}

template <typename T>
T *carve(char *&p, long long n) {
  T *r = reinterpret_cast<T *>(p);
  long long bytes = ((long long)sizeof(T) * std::max(n, 1LL) + 255) & ~255LL;
  p += bytes;
  return r;
}

}  // namespace

// Builds the plan of query blocks [qlo, qhi) against key blocks [klo, khi)
// (qhi / khi < 0: through the last block).
static lc_status plan_create(lc_bsa_plan *out, int T, int H, int W, int block, int local, int stride,
                      int n_cond_frames, int qlo, int qhi, int klo, int khi, void *stream) {
  if (!out || T <= 0 || H <= 0 || W <= 0 || local < 0 || n_cond_frames < 0 ||
      n_cond_frames >= T || block <= 0)
    return LC_ERR_INVALID_ARGUMENT;
  if (block != LC_BLOCK) return LC_ERR_UNSUPPORTED;
  long long N = (long long)T * H * W;
  // Position decoding uses exact multiply-shift division, valid for token
  // indices below 2^24 and frame sizes below 2^16.
  if (N >= (1LL << 24) || (long long)H * W >= (1LL << 16)) return LC_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  lc_bsa_plan_s *p = new (std::nothrow) lc_bsa_plan_s();
  if (!p) return LC_ERR_OUT_OF_MEMORY;
  p->T = T; p->H = H; p->W = W; p->block = block; p->local = local; p->stride = stride;
  p->n_cond = n_cond_frames;
  p->Nc = n_cond_frames * H * W;
  p->Nn = (T - n_cond_frames) * H * W;
  p->Cb = (p->Nc + block - 1) / block;
  p->Nb = (p->Nn + block - 1) / block;
  p->nq = p->Cb + p->Nb;
  p->gc = (p->Cb + 3) / 4;
  p->gn = (p->Nb + 3) / 4;
  p->G = p->gc + p->gn;
  p->kgc = (p->Cb + 1) / 2;
  if (stride > 1) {  // global blocks pair with each other, the others in order
    const int n_glob = (p->Nb + stride - 1) / stride;
    p->kgn = (n_glob + 1) / 2 + (p->Nb - n_glob + 1) / 2;
  } else {
    p->kgn = (p->Nb + 1) / 2;
  }
  p->KG = p->kgc + p->kgn;
  if (qhi < 0) qhi = p->nq;
  if (khi < 0) khi = p->nq;
  if (qlo < 0 || klo < 0 || qlo > qhi || klo > khi || qhi > p->nq || khi > p->nq) {
    delete p;
    return LC_ERR_INVALID_ARGUMENT;
  }
  // Shard query ranges start and end on group boundaries (4 blocks within a
  // segment, or a segment end), so every group lies wholly inside or outside.
  auto group_edge = [&](int b) {
    return b == p->Cb || b == p->nq || (b < p->Cb ? b % 4 == 0 : (b - p->Cb) % 4 == 0);
  };
  if (!group_edge(qlo) || !group_edge(qhi)) {
    delete p;
    return LC_ERR_INVALID_ARGUMENT;
  }
  p->qlo = qlo; p->qhi = qhi; p->klo = klo; p->khi = khi;
  PlanGeom g{p->Nc, p->Nn, p->Cb, p->Nb, p->nq, p->gc, p->gn, p->G, local, stride,
             p->kgc, p->kgn, p->KG, qlo, qhi, klo, khi};
  long long nnz = 0;
  p->G_active = p->G;
  p->fill_needed = false;
  if (qlo == 0 && qhi == p->nq && klo == 0 && khi == p->nq) {  // closed form
    nnz = (long long)p->Cb * p->Cb + (long long)p->Nb * p->Cb;
    for (long long i = 0; i < p->Nb; ++i) nnz += noisy_row_count(i, p->Nb, local, stride);
  } else {  // a shard: count on the host (block pairs; groups with any pair)
    p->G_active = 0;
    for (int gi = 0; gi < p->G; ++gi) {
      const int first = gi < p->gc ? 4 * gi : p->Cb + 4 * (gi - p->gc);
      const int cnt = gi < p->gc ? std::min(4, p->Cb - 4 * gi) : std::min(4, p->Nb - 4 * (gi - p->gc));
      bool any = false;
      for (int r = first; r < first + cnt; ++r) {
        if (r < qlo || r >= qhi) continue;
        for (int c = klo; c < khi; ++c)
          if (attends(r, c, g)) {
            ++nnz;
            any = true;
          }
      }
      p->G_active += any ? 1 : 0;
      if (!any && first >= qlo && first < qhi) p->fill_needed = true;
    }
  }
  p->nnz = nnz;
  if (nnz >= (1LL << 31)) { delete p; return LC_ERR_INVALID_ARGUMENT; }

  lc_status s = lc_from_cuda(cudaGetDevice(&p->device));
  if (s != LC_OK) { delete p; return s; }
  // Size the single allocation (each piece rounded to 256 bytes).
  char *probe = nullptr;
  carve<int>(probe, p->nq + 1); carve<int>(probe, nnz); carve<int>(probe, p->nq);
  carve<int>(probe, p->G + 1); carve<int>(probe, p->G); carve<uint32_t>(probe, nnz);
  carve<int>(probe, p->G); carve<unsigned long long>(probe, 2); carve<int>(probe, 1);
  carve<int>(probe, p->nq + 1); carve<int>(probe, nnz); carve<int>(probe, p->nq);
  carve<int>(probe, p->KG + 1); carve<int>(probe, p->KG); carve<uint32_t>(probe, nnz);
  carve<int>(probe, p->KG); carve<int2>(probe, p->KG); carve<int>(probe, 2);
  size_t bytes = reinterpret_cast<size_t>(probe);
  cudaError_t e = cudaMallocAsync(&p->mem, bytes, st);
  if (e != cudaSuccess) { delete p; return lc_from_cuda(e); }
  char *q = static_cast<char *>(p->mem);
  p->row_ptr = carve<int>(q, p->nq + 1);
  p->col_idx = carve<int>(q, nnz);
  p->row_cnt = carve<int>(q, p->nq);
  p->grp_ptr = carve<int>(q, p->G + 1);
  p->grp_cnt = carve<int>(q, p->G);
  p->grp_ent = carve<uint32_t>(q, nnz);
  p->grp_order = carve<int>(q, p->G);
  p->pairs = carve<unsigned long long>(q, 2);
  p->err = carve<int>(q, 1);
  p->col_ptr = carve<int>(q, p->nq + 1);
  p->row_idx = carve<int>(q, nnz);
  p->col_cnt = carve<int>(q, p->nq);
  p->kgrp_ptr = carve<int>(q, p->KG + 1);
  p->kgrp_cnt = carve<int>(q, p->KG);
  p->kgrp_ent = carve<uint32_t>(q, nnz);
  p->kgrp_order = carve<int>(q, p->KG);
  p->kgrp_blk = carve<int2>(q, p->KG);
  p->sched = carve<int>(q, 2);

  e = cudaMemsetAsync(p->pairs, 0, 2 * sizeof(unsigned long long), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(p->err, 0, sizeof(int), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(p->sched, 0, 2 * sizeof(int), st);
  const int tpb = 256;
  int row_blocks = (p->nq * 32 + tpb - 1) / tpb;
  int grp_blocks = (p->G * 32 + tpb - 1) / tpb;
  int kgrp_blocks = (p->KG * 32 + tpb - 1) / tpb;
  if (e == cudaSuccess) {
    row_scan_kernel<<<row_blocks, tpb, 0, st>>>(g, p->row_cnt, p->pairs);
    group_count_kernel<<<grp_blocks, tpb, 0, st>>>(g, p->grp_cnt);
    col_scan_kernel<<<row_blocks, tpb, 0, st>>>(g, p->col_cnt);
    kgroup_count_kernel<<<kgrp_blocks, tpb, 0, st>>>(g, p->kgrp_cnt);
    kgroup_blocks_kernel<<<(p->KG + 127) / 128, 128, 0, st>>>(g, p->kgrp_blk);
    scan_kernel<<<1, 1024, 0, st>>>(g, p->row_cnt, p->row_ptr, p->grp_cnt, p->grp_ptr,
                                    p->col_cnt, p->col_ptr, p->kgrp_cnt, p->kgrp_ptr, nnz, p->err);
    col_fill_kernel<<<row_blocks, tpb, 0, st>>>(g, p->col_ptr, p->row_idx, nnz, p->err);
    row_fill_kernel<<<row_blocks, tpb, 0, st>>>(g, p->row_ptr, p->col_idx, nnz, p->err);
    group_fill_kernel<<<grp_blocks, tpb, 0, st>>>(g, p->grp_ptr, p->grp_ent, nnz, p->err);
    order_kernel<<<(p->G + 127) / 128, 128, 0, st>>>(p->G, p->grp_cnt, p->grp_order);
    kgroup_fill_kernel<<<kgrp_blocks, tpb, 0, st>>>(g, p->kgrp_ptr, p->kgrp_ent, nnz, p->err);
    order_kernel<<<(p->KG + 127) / 128, 128, 0, st>>>(p->KG, p->kgrp_cnt, p->kgrp_order);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p->ready, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventRecord(p->ready, st);
  if (e != cudaSuccess) {
    cudaFreeAsync(p->mem, st);
    delete p;
    return lc_from_cuda(e);
  }
  *out = p;
  return LC_OK;
}

extern "C" lc_status lc_bsa_plan_create(lc_bsa_plan *out, int T, int H, int W, int block,
                                        int local, int stride, int n_cond_frames, void *stream) {
  return plan_create(out, T, H, W, block, local, stride, n_cond_frames, 0, -1, 0, -1, stream);
}

extern "C" lc_status lc_bsa_plan_create_shard(lc_bsa_plan *out, int T, int H, int W, int block,
                                              int local, int stride, int n_cond_frames,
                                              int q_block_lo, int q_block_hi, int k_block_lo,
                                              int k_block_hi, void *stream) {
  if (q_block_hi < 0 || k_block_hi < 0) return LC_ERR_INVALID_ARGUMENT;
  return plan_create(out, T, H, W, block, local, stride, n_cond_frames, q_block_lo, q_block_hi,
                     k_block_lo, k_block_hi, stream);
}

extern "C" lc_status lc_bsa_plan_token_range(lc_bsa_plan plan, long long *q_lo, long long *q_hi,
                                             long long *k_lo, long long *k_hi) {
  if (!plan || !q_lo || !q_hi || !k_lo || !k_hi) return LC_ERR_INVALID_ARGUMENT;
  *q_lo = lc_block_token(plan, plan->qlo);
  *q_hi = lc_block_token(plan, plan->qhi);
  *k_lo = lc_block_token(plan, plan->klo);
  *k_hi = lc_block_token(plan, plan->khi);
  return LC_OK;
}

extern "C" lc_status lc_bsa_plan_destroy(lc_bsa_plan plan, void *stream) {
  if (!plan) return LC_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaFreeAsync(plan->mem, st);
  cudaEventDestroy(plan->ready);
  delete plan;
  return lc_from_cuda(e);
}

extern "C" lc_status lc_bsa_plan_info(lc_bsa_plan plan, lc_bsa_plan_info_t *info) {
  if (!plan || !info) return LC_ERR_INVALID_ARGUMENT;
  if (!plan->info_cached) {
    LC_CUDA_TRY(cudaEventSynchronize(plan->ready));
    unsigned long long pr[2];
    int err = 0;
    LC_CUDA_TRY(cudaMemcpy(pr, plan->pairs, sizeof(pr), cudaMemcpyDeviceToHost));
    LC_CUDA_TRY(cudaMemcpy(&err, plan->err, sizeof(int), cudaMemcpyDeviceToHost));
    if (err) return LC_ERR_DEVICE_CHECK;
    plan->pairs_host[0] = (long long)pr[0];
    plan->pairs_host[1] = (long long)pr[1];
    plan->info_cached = true;
  }
  info->num_q_blocks = plan->nq;
  info->num_cond_blocks = plan->Cb;
  info->num_noisy_blocks = plan->Nb;
  info->nnz = plan->nnz;
  info->n_cond_tokens = plan->Nc;
  info->n_noisy_tokens = plan->Nn;
  info->attended_token_pairs = plan->pairs_host[0];
  info->attended_token_pairs_noisy = plan->pairs_host[1];
  return LC_OK;
}

extern "C" lc_status lc_bsa_plan_copy_csc(lc_bsa_plan plan, int *col_ptr_host, int *row_idx_host,
                                          void *stream) {
  if (!plan || !col_ptr_host || !row_idx_host) return LC_ERR_INVALID_ARGUMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  LC_CUDA_TRY(cudaStreamWaitEvent(st, plan->ready, 0));
  LC_CUDA_TRY(cudaMemcpyAsync(col_ptr_host, plan->col_ptr, sizeof(int) * (plan->nq + 1),
                              cudaMemcpyDeviceToHost, st));
  LC_CUDA_TRY(cudaMemcpyAsync(row_idx_host, plan->row_idx, sizeof(int) * plan->nnz,
                              cudaMemcpyDeviceToHost, st));
  int err = 0;
  LC_CUDA_TRY(cudaMemcpyAsync(&err, plan->err, sizeof(int), cudaMemcpyDeviceToHost, st));
  LC_CUDA_TRY(cudaStreamSynchronize(st));
  return err ? LC_ERR_DEVICE_CHECK : LC_OK;
}

extern "C" lc_status lc_bsa_plan_copy_csr(lc_bsa_plan plan, int *row_ptr_host, int *col_idx_host,
                                          void *stream) {
  if (!plan || !row_ptr_host || !col_idx_host) return LC_ERR_INVALID_ARGUMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  LC_CUDA_TRY(cudaStreamWaitEvent(st, plan->ready, 0));
  LC_CUDA_TRY(cudaMemcpyAsync(row_ptr_host, plan->row_ptr, sizeof(int) * (plan->nq + 1),
                              cudaMemcpyDeviceToHost, st));
  LC_CUDA_TRY(cudaMemcpyAsync(col_idx_host, plan->col_idx, sizeof(int) * plan->nnz,
                              cudaMemcpyDeviceToHost, st));
  int err = 0;
  LC_CUDA_TRY(cudaMemcpyAsync(&err, plan->err, sizeof(int), cudaMemcpyDeviceToHost, st));
  LC_CUDA_TRY(cudaStreamSynchronize(st));
  return err ? LC_ERR_DEVICE_CHECK : LC_OK;
}
