// attn_sm100.cu -- bf16 block-sparse 3D-RoPE attention on B200 tensor cores.
//
// What it computes: for every query token, softmax over its attended keys of
// scale * <R(q), R(k)>, times v, with R the partitioned 3D-RoPE
// ("longcat-video-rs" header card and section 03-01) and the attended keys
// given by the local + strided-global block pattern with condition tokens
// isolated from noise tokens ("longcat-video-rs" section 03-03; myzaker /
// QbitAI "背后技术原理").  Inside a block the attention is dense, across
// blocks it is sparse (zhichai.net "Block Sparse Attention").
//
// How (one persistent CTA per SM, 12 warps):
//   work item = (batch, head, group of up to 4 query blocks of one segment),
//               handed out by an atomic counter in longest-list-first order;
//               its two 128-row query tiles Q0, Q1 share one key list, the
//               sorted union of the member blocks' lists, walked two key
//               blocks (128 keys) at a time.
//   warp 8      TMA producer: Q tiles, then the listed K and V blocks into a
//               3-stage ring (missing second block = out-of-range box, which
//               TMA fills with zeros).
//   warps 10-11 RoPE: rotate every freshly loaded Q and K tile in shared
//               memory (128-byte swizzled rows, cos/sin tables in smem).
//   warp 9      MMA issuer (one thread): S_i = Q_i K^T (M=128, N=128, K=64)
//               into TMEM, O_i += P_i V (A = P from TMEM, M=128, N=64).
//   warps 0-3 / 4-7  softmax of Q0 / Q1, one TMEM lane (= query row) per
//               thread: mask, running max with lazy rescaling (threshold 2^8),
//               exp2, row sum, P as bf16 into TMEM; at the end O / l through
//               shared memory to a TMA store, plus the log-sum-exp.
//   TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,320) O1 [320,384)
//               P0 [384,448) P1 [448,512).
// Every wait on an mbarrier is bounded (globaltimer); on expiry the kernel
// flags LC_DEVSTAT_TIMEOUT in the device status word, stops all roles of the
// CTA, drains its own copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include <string.h>

#include <mutex>

#include "lc_internal.cuh"
#include "sm100_ptx.cuh"

namespace {

constexpr int kStages = 3;
constexpr int kThreads = 384;
constexpr int kWarpProducer = 8;
constexpr int kWarpMma = 9;
constexpr int kWarpRope = 10;  // and 11
constexpr int kRopeThreads = 64;
constexpr int kTileBytes = 128 * 128;  // 128 rows x 64 bf16
constexpr int kBoxBytes = 64 * 128;    // one 64-row TMA box
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 320, kColP0 = 384,
                   kColP1 = 448;
constexpr uint32_t kIdescQK = lcptx::idesc_bf16_f32(128, 128, 0, 0);
constexpr uint32_t kIdescPV = lcptx::idesc_bf16_f32(128, 64, 0, 1);
constexpr float kRescaleThreshold = 8.0f;  // log2 units: p stays below 2^8 before a rescale

struct __align__(64) Sm100Params {
  CUtensorMap tmQ[2], tmK[2], tmV[2], tmO[2];  // [0] condition segment, [1] noisy segment
  const float *rope_tab;
  const int *grp_ptr;
  const uint32_t *grp_ent;
  const int *grp_order;
  int *work_counter;
  int *status;
  float *lse;
  long long timeout_ns;
  lc_divmod div_hw, div_w;
  int T, H, W;
  int Nc, Nn, Cb, gc;
  int heads, n_groups_active, total_items;
  int lse_nq;          // rows of the lse tensor per (batch, head)
  int q_row_offset_noisy;  // row of the q/out/lse tensors holding noisy token 0
  int tab_floats;
  float scale_log2;
};

// Shared memory carve-up (offsets from a 1024-aligned base).
struct SmemOffsets {
  static constexpr int q = 0;                                  // 2 tiles
  static constexpr int k = q + 2 * kTileBytes;                 // kStages tiles
  static constexpr int v = k + kStages * kTileBytes;           // kStages tiles
  static constexpr int bars = v + kStages * kTileBytes;        // mbarriers
  static constexpr int n_bars = 64;
  static constexpr int misc = bars + n_bars * 8;               // tmem base, items, abort
  static constexpr int tab = misc + 64;                        // rope tables (fp32)
};

// Barrier indices.
enum {
  B_QFULL = 0,   // [2] TMA Q landed
  B_QREADY = 2,  // [2] Q rotated
  B_QEMPTY = 4,  // [2] Q buffer (and O staging) free
  B_KFULL = 6,   // [kStages]
  B_KREADY = 6 + kStages,
  B_KEMPTY = 6 + 2 * kStages,
  B_VFULL = 6 + 3 * kStages,
  B_VEMPTY = 6 + 4 * kStages,
  B_SFULL = 6 + 5 * kStages,  // [2]
  B_SFREE = B_SFULL + 2,      // [2]
  B_PFULL = B_SFREE + 2,      // [2]
  B_ODONE = B_PFULL + 2,      // [2]
  B_EPI = B_ODONE + 2,        // [2] O rows staged in smem
  B_SCHED_FULL = B_EPI + 2,   // [2]
  B_SCHED_EMPTY = B_SCHED_FULL + 2,  // [2]
  B_DRAIN = B_SCHED_EMPTY + 2,
  B_COUNT = B_DRAIN + 1
};
static_assert(B_COUNT <= SmemOffsets::n_bars, "barrier space");
constexpr int kSchedConsumers = 8 + 1 + 2;  // softmax warps, MMA warp, RoPE warps

struct Ctx {
  uint32_t bar0;                 // smem address of barrier 0
  volatile int *abort_flag;      // smem
  int *status;
  long long timeout_ns;
  __device__ uint32_t bar(int i) const { return bar0 + 8u * (uint32_t)i; }
};

// Bounded wait: true when the phase of `parity` completed; false when the CTA
// aborted or this wait timed out (which sets the abort flag and the status).
__device__ __noinline__ bool wait_bar(const Ctx &c, uint32_t bar, uint32_t parity) {
  if (lcptx::mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = lcptx::globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (lcptx::mbar_try_wait(bar, parity)) return true;
    if ((it & 31u) == 0) {
      if (*c.abort_flag) return false;
      if ((long long)(lcptx::globaltimer_ns() - t0) > c.timeout_ns) {
        atomicOr(c.status, LC_DEVSTAT_TIMEOUT);
        *c.abort_flag = 1;
        __threadfence_block();
        return false;
      }
    }
  }
}

// Warp-uniform form for warps whose lanes then run .sync.aligned tcgen05 ops
// together: every lane waits, and the warp fails as one if any lane failed.
__device__ __forceinline__ bool wait_warp(const Ctx &c, uint32_t bar, uint32_t parity) {
  return __all_sync(0xffffffffu, wait_bar(c, bar, parity)) != 0;
}

struct Item {
  int b, h, seg, row0, seg_len, len;
  const uint32_t *ent;
};

__device__ __forceinline__ Item decode_item(const Sm100Params &p, int item) {
  Item it;
  int per = p.n_groups_active;
  int bh = item / per;
  int g = p.grp_order[item - bh * per];
  it.b = bh / p.heads;
  it.h = bh - it.b * p.heads;
  it.seg = g < p.gc ? 0 : 1;
  int qb0 = it.seg ? 4 * (g - p.gc) : 4 * g;
  it.row0 = 64 * qb0;
  it.seg_len = it.seg ? p.Nn : p.Nc;
  int lo = p.grp_ptr[g];
  it.len = p.grp_ptr[g + 1] - lo;
  it.ent = p.grp_ent + lo;
  return it;
}

// Key block `e` (plan entry) -> segment, first token in the segment, token count.
__device__ __forceinline__ void entry_block(const Sm100Params &p, uint32_t e, int &seg, int &row,
                                            int &cnt) {
  int c = (int)(e & 0xFFFFFFu);
  if (c < p.Cb) {
    seg = 0;
    row = 64 * c;
    cnt = min(64, p.Nc - row);
  } else {
    seg = 1;
    row = 64 * (c - p.Cb);
    cnt = min(64, p.Nn - row);
  }
}

__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// Rotate rows [r_begin, r_end) of a swizzled 64-channel bf16 tile in place;
// tile row r holds sequence token tok0 + r.  Threads of the RoPE warps split
// the (row, 16-byte chunk) pairs.
__device__ __forceinline__ void rope_tile(uint8_t *tile, int r_begin, int r_end, int tok0,
                                          const float *tab, const Sm100Params &p, int rt) {
  const float *cT = tab, *sT = tab + p.T * 8;
  const float *cH = sT + p.T * 8, *sH = cH + p.H * 12;
  const float *cW = sH + p.H * 12, *sW = cW + p.W * 12;
  const int jobs = (r_end - r_begin) * 8;
  for (int j = rt; j < jobs; j += kRopeThreads) {
    int r = r_begin + (j >> 3), ch = j & 7;
    int n = tok0 + r;
    int t = lc_div(n, p.div_hw);
    int rem = n - t * p.div_hw.d;
    int hh = lc_div(rem, p.div_w);
    int w = rem - hh * p.div_w.d;
    const float *c, *s;
    if (ch < 2) { c = cT + t * 8 + 4 * ch; s = sT + t * 8 + 4 * ch; }
    else if (ch < 5) { c = cH + hh * 12 + 4 * (ch - 2); s = sH + hh * 12 + 4 * (ch - 2); }
    else { c = cW + w * 12 + 4 * (ch - 5); s = sW + w * 12 + 4 * (ch - 5); }
    float4 cc = *reinterpret_cast<const float4 *>(c);
    float4 ss = *reinterpret_cast<const float4 *>(s);
    uint4 *ptr = reinterpret_cast<uint4 *>(tile + swz(r, ch));
    uint4 raw = *ptr;
    uint32_t wds[4] = {raw.x, raw.y, raw.z, raw.w};
    const float cs[4] = {cc.x, cc.y, cc.z, cc.w}, sn[4] = {ss.x, ss.y, ss.z, ss.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      __nv_bfloat162 v2 = *reinterpret_cast<__nv_bfloat162 *>(&wds[q]);
      float2 f = __bfloat1622float2(v2);
      float a = f.x * cs[q] - f.y * sn[q];
      float b = f.x * sn[q] + f.y * cs[q];
      __nv_bfloat162 o2 = __floats2bfloat162_rn(a, b);
      wds[q] = *reinterpret_cast<uint32_t *>(&o2);
    }
    *ptr = make_uint4(wds[0], wds[1], wds[2], wds[3]);
  }
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

__global__ void __launch_bounds__(kThreads, 1) bsa_sm100_kernel(const __grid_constant__ Sm100Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  uint8_t *sQ = smem + SmemOffsets::q;
  uint8_t *sK = smem + SmemOffsets::k;
  uint8_t *sV = smem + SmemOffsets::v;
  uint32_t *misc = reinterpret_cast<uint32_t *>(smem + SmemOffsets::misc);
  // misc[0] tmem base, misc[1..2] scheduled items, misc[3] abort flag
  float *tab = reinterpret_cast<float *>(smem + SmemOffsets::tab);
  Ctx ctx;
  ctx.bar0 = lcptx::smem_addr(smem + SmemOffsets::bars);
  ctx.abort_flag = reinterpret_cast<volatile int *>(&misc[3]);
  ctx.status = p.status;
  ctx.timeout_ns = p.timeout_ns;

  // ---- set-up: tables, barriers, TMEM
  for (int i = tid; i < p.tab_floats; i += kThreads) tab[i] = p.rope_tab[i];
  if (tid == 0) {
    misc[3] = 0;
    for (int i = 0; i < 2; ++i) {
      lcptx::mbar_init(ctx.bar(B_QFULL + i), 1);
      lcptx::mbar_init(ctx.bar(B_QREADY + i), kRopeThreads);
      lcptx::mbar_init(ctx.bar(B_QEMPTY + i), 1);
      lcptx::mbar_init(ctx.bar(B_SFULL + i), 1);
      lcptx::mbar_init(ctx.bar(B_SFREE + i), 4);
      lcptx::mbar_init(ctx.bar(B_PFULL + i), 4);
      lcptx::mbar_init(ctx.bar(B_ODONE + i), 1);
      lcptx::mbar_init(ctx.bar(B_EPI + i), 128);
      lcptx::mbar_init(ctx.bar(B_SCHED_FULL + i), 1);
      lcptx::mbar_init(ctx.bar(B_SCHED_EMPTY + i), kSchedConsumers);
    }
    for (int s = 0; s < kStages; ++s) {
      lcptx::mbar_init(ctx.bar(B_KFULL + s), 1);
      lcptx::mbar_init(ctx.bar(B_KREADY + s), kRopeThreads);
      lcptx::mbar_init(ctx.bar(B_KEMPTY + s), 1);
      lcptx::mbar_init(ctx.bar(B_VFULL + s), 1);
      lcptx::mbar_init(ctx.bar(B_VEMPTY + s), 1);
    }
    lcptx::mbar_init(ctx.bar(B_DRAIN), 1);
    lcptx::fence_mbar_init();
  }
  if (warp == kWarpMma) {
    lcptx::tmem_alloc(lcptx::smem_addr(&misc[0]), kTmemCols);
    lcptx::tmem_relinquish();
  }
  if (warp == kWarpProducer && lane == 0) {
    for (int i = 0; i < 2; ++i) {
      lcptx::tma_prefetch_desc(&p.tmQ[i]);
      lcptx::tma_prefetch_desc(&p.tmK[i]);
      lcptx::tma_prefetch_desc(&p.tmV[i]);
      lcptx::tma_prefetch_desc(&p.tmO[i]);
    }
  }
  lcptx::tc_fence_before();
  __syncthreads();
  lcptx::tc_fence_after();
  const uint32_t tmem = misc[0];

  if (warp == kWarpProducer) {
    // ======================= TMA producer (one thread) =======================
    if (lane == 0) {
      uint32_t kv_it = 0, item_it = 0;
      uint32_t k_issued[kStages], v_issued[kStages], q_issued[2] = {0xFFFFFFFFu, 0xFFFFFFFFu};
      for (int s = 0; s < kStages; ++s) k_issued[s] = v_issued[s] = 0xFFFFFFFFu;
      for (;;) {
        const int slot = item_it & 1;
        const uint32_t sph = (item_it >> 1) & 1;
        int item = atomicAdd(p.work_counter, 1);
        if (item >= p.total_items) item = -1;
        if (!wait_bar(ctx, ctx.bar(B_SCHED_EMPTY + slot), sph ^ 1)) break;
        misc[1 + slot] = (uint32_t)item;
        lcptx::mbar_arrive(ctx.bar(B_SCHED_FULL + slot));
        if (item < 0) break;
        const Item it = decode_item(p, item);
        bool ok = true;
        for (int i = 0; i < 2 && ok; ++i) {
          ok = wait_bar(ctx, ctx.bar(B_QEMPTY + i), (item_it & 1) ^ 1);
          if (!ok) break;
          uint32_t bq = ctx.bar(B_QFULL + i);
          lcptx::mbar_arrive_expect_tx(bq, kTileBytes);
          uint32_t dst = lcptx::smem_addr(sQ + i * kTileBytes);
          int r = it.row0 + 128 * i;
          lcptx::tma_load_4d(dst, &p.tmQ[it.seg], bq, 0, it.h, r, it.b);
          lcptx::tma_load_4d(dst + kBoxBytes, &p.tmQ[it.seg], bq, 0, it.h, r + 64, it.b);
          q_issued[i] = item_it & 1;
        }
        if (!ok) break;
        const int ntiles = (it.len + 1) >> 1;
        for (int t = 0; t < ntiles && ok; ++t, ++kv_it) {
          const int s = kv_it % kStages;
          const uint32_t ph = (kv_it / kStages) & 1;
          int sa, ra, na, sb, rb, nb;
          entry_block(p, it.ent[2 * t], sa, ra, na);
          if (2 * t + 1 < it.len) {
            entry_block(p, it.ent[2 * t + 1], sb, rb, nb);
          } else {  // no second block: a box entirely past the segment end reads zeros
            sb = 1;
            rb = p.Nn;
          }
          ok = wait_bar(ctx, ctx.bar(B_KEMPTY + s), ph ^ 1);
          if (!ok) break;
          uint32_t bk = ctx.bar(B_KFULL + s);
          lcptx::mbar_arrive_expect_tx(bk, kTileBytes);
          uint32_t dk = lcptx::smem_addr(sK + s * kTileBytes);
          lcptx::tma_load_4d(dk, &p.tmK[sa], bk, 0, it.h, ra, it.b);
          lcptx::tma_load_4d(dk + kBoxBytes, &p.tmK[sb], bk, 0, it.h, rb, it.b);
          k_issued[s] = ph;
          ok = wait_bar(ctx, ctx.bar(B_VEMPTY + s), ph ^ 1);
          if (!ok) break;
          uint32_t bv = ctx.bar(B_VFULL + s);
          lcptx::mbar_arrive_expect_tx(bv, kTileBytes);
          uint32_t dv = lcptx::smem_addr(sV + s * kTileBytes);
          lcptx::tma_load_4d(dv, &p.tmV[sa], bv, 0, it.h, ra, it.b);
          lcptx::tma_load_4d(dv + kBoxBytes, &p.tmV[sb], bv, 0, it.h, rb, it.b);
          v_issued[s] = ph;
        }
        if (!ok) break;
        ++item_it;
      }
      // Drain: every load this thread issued must land before the CTA exits.
      for (int i = 0; i < 2; ++i) {
        if (q_issued[i] != 0xFFFFFFFFu) {
          uint64_t t0 = lcptx::globaltimer_ns();
          while (!lcptx::mbar_try_wait(ctx.bar(B_QFULL + i), q_issued[i]) &&
                 (long long)(lcptx::globaltimer_ns() - t0) < p.timeout_ns) {}
        }
      }
      for (int s = 0; s < kStages; ++s) {
        if (k_issued[s] != 0xFFFFFFFFu) {
          uint64_t t0 = lcptx::globaltimer_ns();
          while (!lcptx::mbar_try_wait(ctx.bar(B_KFULL + s), k_issued[s]) &&
                 (long long)(lcptx::globaltimer_ns() - t0) < p.timeout_ns) {}
        }
        if (v_issued[s] != 0xFFFFFFFFu) {
          uint64_t t0 = lcptx::globaltimer_ns();
          while (!lcptx::mbar_try_wait(ctx.bar(B_VFULL + s), v_issued[s]) &&
                 (long long)(lcptx::globaltimer_ns() - t0) < p.timeout_ns) {}
        }
      }
    }
  } else if (warp == kWarpMma) {
    // ======================= MMA issuer (one thread) =========================
    uint32_t item_it = 0, kv_it = 0;
    uint32_t sfree_ph[2] = {0, 0}, pfull_ph[2] = {0, 0};
    if (lane == 0) for (;;) {
      const int slot = item_it & 1;
      if (!wait_bar(ctx, ctx.bar(B_SCHED_FULL + slot), (item_it >> 1) & 1)) break;
      const int item = (int)misc[1 + slot];
      lcptx::mbar_arrive(ctx.bar(B_SCHED_EMPTY + slot));
      if (item < 0) break;
      const Item it = decode_item(p, item);
      const int ntiles = (it.len + 1) >> 1;
      bool ok = wait_bar(ctx, ctx.bar(B_QREADY + 0), item_it & 1) &&
                wait_bar(ctx, ctx.bar(B_QREADY + 1), item_it & 1);
      if (!ok) break;
      const uint32_t q_addr[2] = {lcptx::smem_addr(sQ), lcptx::smem_addr(sQ + kTileBytes)};
      auto issue_s = [&](int i, int s) -> bool {
        if (!wait_bar(ctx, ctx.bar(B_SFREE + i), sfree_ph[i] ^ 1)) return false;
        sfree_ph[i] ^= 1;
        lcptx::tc_fence_after();
        const uint32_t kb = lcptx::smem_addr(sK + s * kTileBytes);
        const uint32_t d = tmem + (i ? kColS1 : kColS0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          uint64_t a = lcptx::smem_desc_sw128(q_addr[i] + 32 * kk, 16, 1024);
          uint64_t b = lcptx::smem_desc_sw128(kb + 32 * kk, 16, 1024);
          lcptx::mma_ss(d, a, b, kIdescQK, kk > 0);
        }
        lcptx::mma_commit(ctx.bar(B_SFULL + i));
        return true;
      };
      auto issue_pv = [&](int i, int s, bool accumulate) -> bool {
        if (!wait_bar(ctx, ctx.bar(B_PFULL + i), pfull_ph[i])) return false;
        pfull_ph[i] ^= 1;
        lcptx::tc_fence_after();
        const uint32_t vb = lcptx::smem_addr(sV + s * kTileBytes);
        const uint32_t d = tmem + (i ? kColO1 : kColO0);
        const uint32_t a = tmem + (i ? kColP1 : kColP0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          uint64_t b = lcptx::smem_desc_sw128(vb + 2048 * kk, 8192, 1024);
          lcptx::mma_ts(d, a + 8 * kk, b, kIdescPV, (accumulate || kk > 0) ? 1u : 0u);
        }
        lcptx::mma_commit(ctx.bar(B_ODONE + i));
        return true;
      };
      // Tile 0: both S tiles.
      {
        const int s = kv_it % kStages;
        ok = wait_bar(ctx, ctx.bar(B_KREADY + s), (kv_it / kStages) & 1) && issue_s(0, s) &&
             issue_s(1, s);
        if (!ok) break;
        lcptx::mma_commit(ctx.bar(B_KEMPTY + s));
      }
      for (int t = 0; t < ntiles && ok; ++t) {
        const uint32_t cur = kv_it + t;
        const int s = cur % kStages;
        const bool more = t + 1 < ntiles;
        const int s_next = (cur + 1) % kStages;
        if (more) {
          ok = wait_bar(ctx, ctx.bar(B_KREADY + s_next), ((cur + 1) / kStages) & 1) &&
               issue_s(0, s_next);
          if (!ok) break;
        }
        ok = wait_bar(ctx, ctx.bar(B_VFULL + s), (cur / kStages) & 1) && issue_pv(0, s, t > 0);
        if (!ok) break;
        if (more) {
          ok = issue_s(1, s_next);
          if (!ok) break;
          lcptx::mma_commit(ctx.bar(B_KEMPTY + s_next));
        }
        ok = issue_pv(1, s, t > 0);
        if (!ok) break;
        lcptx::mma_commit(ctx.bar(B_VEMPTY + s));
      }
      if (!ok) break;
      kv_it += ntiles;
      ++item_it;
    }
    if (lane == 0) {
      // Drain: wait until every MMA this thread issued has completed.
      lcptx::mma_commit(ctx.bar(B_DRAIN));
      uint64_t t0 = lcptx::globaltimer_ns();
      while (!lcptx::mbar_try_wait(ctx.bar(B_DRAIN), 0) &&
             (long long)(lcptx::globaltimer_ns() - t0) < p.timeout_ns) {}
    }
    __syncwarp();
  } else if (warp >= kWarpRope) {
    // ======================= RoPE warps ======================================
    const int rt = tid - kWarpRope * 32;
    uint32_t item_it = 0, kv_it = 0;
    for (;;) {
      const int slot = item_it & 1;
      if (!wait_warp(ctx, ctx.bar(B_SCHED_FULL + slot), (item_it >> 1) & 1)) break;
      const int item = (int)misc[1 + slot];
      __syncwarp();
      if (lane == 0) lcptx::mbar_arrive(ctx.bar(B_SCHED_EMPTY + slot));
      if (item < 0) break;
      const Item it = decode_item(p, item);
      const int seg_base = it.seg ? p.Nc : 0;  // sequence index of the segment's token 0
      bool ok = true;
      for (int i = 0; i < 2 && ok; ++i) {
        ok = wait_warp(ctx, ctx.bar(B_QFULL + i), item_it & 1);
        if (!ok) break;
        int r0 = it.row0 + 128 * i;
        int nrows = min(128, it.seg_len - r0);
        if (nrows > 0) rope_tile(sQ + i * kTileBytes, 0, nrows, seg_base + r0, tab, p, rt);
        lcptx::fence_proxy_async_smem();
        lcptx::mbar_arrive(ctx.bar(B_QREADY + i));
      }
      if (!ok) break;
      const int ntiles = (it.len + 1) >> 1;
      for (int t = 0; t < ntiles; ++t, ++kv_it) {
        const int s = kv_it % kStages;
        ok = wait_warp(ctx, ctx.bar(B_KFULL + s), (kv_it / kStages) & 1);
        if (!ok) break;
        int sa, ra, na;
        entry_block(p, it.ent[2 * t], sa, ra, na);
        uint8_t *tile = sK + s * kTileBytes;
        rope_tile(tile, 0, na, (sa ? p.Nc : 0) + ra, tab, p, rt);
        if (2 * t + 1 < it.len) {
          int sb, rb, nb;
          entry_block(p, it.ent[2 * t + 1], sb, rb, nb);
          rope_tile(tile, 64, 64 + nb, (sb ? p.Nc : 0) + rb - 64, tab, p, rt);
        }
        lcptx::fence_proxy_async_smem();
        lcptx::mbar_arrive(ctx.bar(B_KREADY + s));
      }
      if (!ok) break;
      ++item_it;
    }
  } else {
    // ======================= softmax warpgroups ==============================
    const int wg = warp >> 2;              // which Q tile
    const int row = tid & 127;             // TMEM lane == tile row
    const int qsub = 2 * wg + (row >> 6);  // member index of this row's query block
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + (wg ? kColS1 : kColS0);
    const uint32_t tO = tmem + lane_base + (wg ? kColO1 : kColO0);
    const uint32_t tP = tmem + lane_base + (wg ? kColP1 : kColP0);
    uint32_t item_it = 0, sfull_ph = 0, odone_ph = 0;
    for (;;) {
      const int slot = item_it & 1;
      if (!wait_warp(ctx, ctx.bar(B_SCHED_FULL + slot), (item_it >> 1) & 1)) break;
      const int item = (int)misc[1 + slot];
      __syncwarp();
      if (lane == 0) lcptx::mbar_arrive(ctx.bar(B_SCHED_EMPTY + slot));
      if (item < 0) break;
      const Item it = decode_item(p, item);
      const int ntiles = (it.len + 1) >> 1;
      float m_ref = -INFINITY, l_sum = 0.f;
      bool ok = true;
      for (int t = 0; t < ntiles; ++t) {
        // Mask limits for this warp's rows (uniform across the warp).
        int sa, ra, na, nb = 0;
        uint32_t ea = it.ent[2 * t];
        entry_block(p, ea, sa, ra, na);
        if (!((ea >> (24 + qsub)) & 1u)) na = 0;
        if (2 * t + 1 < it.len) {
          uint32_t eb = it.ent[2 * t + 1];
          int sb, rb;
          entry_block(p, eb, sb, rb, nb);
          if (!((eb >> (24 + qsub)) & 1u)) nb = 0;
        }
        ok = wait_warp(ctx, ctx.bar(B_SFULL + wg), sfull_ph);
        if (!ok) break;
        sfull_ph ^= 1;
        lcptx::tc_fence_after();
        float s[128];
        {
          uint32_t r32[32];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            lcptx::tmem_ld32(tS + 32 * c, r32);
            lcptx::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) s[32 * c + j] = __uint_as_float(r32[j]);
          }
        }
        lcptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) lcptx::mbar_arrive(ctx.bar(B_SFREE + wg));
        if (na < 64) {
#pragma unroll
          for (int j = 0; j < 64; ++j)
            if (j >= na) s[j] = -INFINITY;
        }
        if (nb < 64) {
#pragma unroll
          for (int j = 0; j < 64; ++j)
            if (j >= nb) s[64 + j] = -INFINITY;
        }
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < 128; ++j) mx = fmaxf(mx, s[j]);
        const float mt = mx * p.scale_log2;
        float alpha = 1.f;
        bool rescale_o = false;
        if (t == 0) {
          m_ref = mt;
        } else {
          bool need = mt > m_ref + kRescaleThreshold;
          if (__any_sync(0xffffffffu, need)) {
            float m_new = fmaxf(m_ref, mt);
            alpha = (m_new == -INFINITY) ? 1.f : ex2(m_ref - m_new);
            l_sum *= alpha;
            m_ref = m_new;
            rescale_o = true;
          }
        }
        const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
        uint32_t pk[64];
        float lsum_t = 0.f;
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          float p0 = ex2(fmaf(s[2 * j], p.scale_log2, -m_use));
          float p1 = ex2(fmaf(s[2 * j + 1], p.scale_log2, -m_use));
          lsum_t += p0 + p1;
          pk[j] = pack_bf16(p0, p1);
        }
        l_sum += lsum_t;
        // P and O may be touched only after the previous P*V finished.
        if (t > 0) {
          ok = wait_warp(ctx, ctx.bar(B_ODONE + wg), odone_ph);
          if (!ok) break;
          odone_ph ^= 1;
          lcptx::tc_fence_after();
          if (rescale_o) {
            uint32_t o32[32];
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              lcptx::tmem_ld32(tO + 32 * c, o32);
              lcptx::tmem_wait_ld();
#pragma unroll
              for (int j = 0; j < 32; ++j) o32[j] = __float_as_uint(__uint_as_float(o32[j]) * alpha);
              lcptx::tmem_st32(tO + 32 * c, o32);
            }
          }
        }
        {
          uint32_t h0[32], h1[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) { h0[j] = pk[j]; h1[j] = pk[32 + j]; }
          lcptx::tmem_st32(tP, h0);
          lcptx::tmem_st32(tP + 32, h1);
        }
        lcptx::tmem_wait_st();
        lcptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) lcptx::mbar_arrive(ctx.bar(B_PFULL + wg));
      }
      if (!ok) break;
      // ---- epilogue: O / l -> bf16 -> smem (swizzled) -> TMA store; lse
      ok = wait_warp(ctx, ctx.bar(B_ODONE + wg), odone_ph);
      if (!ok) break;
      odone_ph ^= 1;
      lcptx::tc_fence_after();
      const float inv_l = l_sum > 0.f ? 1.f / l_sum : 0.f;
      uint8_t *stage = sQ + wg * kTileBytes;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t o32[32];
        lcptx::tmem_ld32(tO + 32 * c, o32);
        lcptx::tmem_wait_ld();
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint4 v;
          v.x = pack_bf16(__uint_as_float(o32[8 * ch + 0]) * inv_l, __uint_as_float(o32[8 * ch + 1]) * inv_l);
          v.y = pack_bf16(__uint_as_float(o32[8 * ch + 2]) * inv_l, __uint_as_float(o32[8 * ch + 3]) * inv_l);
          v.z = pack_bf16(__uint_as_float(o32[8 * ch + 4]) * inv_l, __uint_as_float(o32[8 * ch + 5]) * inv_l);
          v.w = pack_bf16(__uint_as_float(o32[8 * ch + 6]) * inv_l, __uint_as_float(o32[8 * ch + 7]) * inv_l);
          *reinterpret_cast<uint4 *>(stage + swz(row, 4 * c + ch)) = v;
        }
      }
      lcptx::tc_fence_before();
      const int qrow = it.row0 + 128 * wg + row;  // row within the segment
      if (p.lse && qrow < it.seg_len) {
        const int out_row = (it.seg ? p.q_row_offset_noisy : 0) + qrow;
        p.lse[((long long)it.b * p.heads + it.h) * p.lse_nq + out_row] =
            ((m_ref == -INFINITY ? 0.f : m_ref) + __log2f(l_sum)) * 0.69314718055994530942f;
      }
      lcptx::fence_proxy_async_smem();
      lcptx::mbar_arrive(ctx.bar(B_EPI + wg));
      if (row == 0) {
        ok = wait_bar(ctx, ctx.bar(B_EPI + wg), item_it & 1);
        if (ok) {
          const uint32_t src = lcptx::smem_addr(stage);
          const int r0 = it.row0 + 128 * wg;
          if (r0 < it.seg_len)
            lcptx::tma_store_4d(&p.tmO[it.seg], src, 0, it.h, r0, it.b);
          if (r0 + 64 < it.seg_len)
            lcptx::tma_store_4d(&p.tmO[it.seg], src + kBoxBytes, 0, it.h, r0 + 64, it.b);
          lcptx::bulk_commit_group();
          lcptx::bulk_wait_group_read0();
          lcptx::mbar_arrive(ctx.bar(B_QEMPTY + wg));
        }
      }
      if ((warp & 3) == 0) ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      ++item_it;
    }
    if (row == 0) lcptx::bulk_wait_group0();
  }

  // ---- teardown
  lcptx::tc_fence_before();
  __syncthreads();
  lcptx::tc_fence_after();
  if (warp == kWarpMma) lcptx::tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// Tensor map over one segment of a [B, ntot, heads, 64] bf16 tensor: tokens
// [tok0, tok0 + nseg) of every batch entry; boxes of 64 tokens x 1 head.
lc_status encode_segment(CUtensorMap *m, const void *base, int batch, long long ntot,
                         long long tok0, long long nseg, int heads) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return LC_ERR_CUDA;
  const long long row_bytes = (long long)heads * LC_HEAD_DIM * 2;
  void *addr = const_cast<char *>(static_cast<const char *>(base)) + tok0 * row_bytes;
  cuuint64_t dims[4] = {LC_HEAD_DIM, (cuuint64_t)heads, (cuuint64_t)nseg, (cuuint64_t)batch};
  cuuint64_t strides[3] = {LC_HEAD_DIM * 2, (cuuint64_t)row_bytes, (cuuint64_t)(ntot * row_bytes)};
  cuuint32_t box[4] = {LC_HEAD_DIM, 1, 64, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, addr, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? LC_OK : LC_ERR_CUDA;
}

__global__ void watchdog_selftest_kernel(int *status, long long timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    lcptx::mbar_init(lcptx::smem_addr(&bar), 1);
    lcptx::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    Ctx c;
    c.bar0 = lcptx::smem_addr(&bar);
    c.abort_flag = &abort_flag;
    c.status = status;
    c.timeout_ns = timeout_ns;
    wait_bar(c, c.bar(0), 0);  // nothing ever arrives: the wait must give up
  }
}

}  // namespace

// ------------------------------------------------------------ no-alloc scratch
// Fixed device scratch for lc_bsa_forward_noalloc, for callers that must not
// allocate device memory.  Word 0 is the work-item counter of the persistent
// scheduler, word 1 the status word the bounded waits report into; the rest
// is reserved.  Every GPU that loads the library holds these 256 bytes until
// the process exits.  In host code the symbol is only a stand-in, so its
// device address is looked up once per device with cudaGetSymbolAddress.
static __device__ __align__(256) int g_lc_noalloc_scratch[LC_NOALLOC_SCRATCH_INTS];

namespace {
constexpr int kNoallocMaxDevices = 64;
std::mutex g_noalloc_mu;
int *g_noalloc_ptr[kNoallocMaxDevices] = {nullptr};
}  // namespace

int *lc_noalloc_scratch(lc_status *st) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoallocMaxDevices) {
    *st = LC_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void *p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_lc_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      *st = LC_ERR_CUDA;
      return nullptr;
    }
    g_noalloc_ptr[dev] = static_cast<int *>(p);
  }
  *st = LC_OK;
  return g_noalloc_ptr[dev];
}

lc_status lc_launch_forward_sm100(const void *q, const void *k, const void *v, const void *cond_k,
                                  const void *cond_v, void *out, float *lse, int batch, int heads,
                                  float scale, bool cached, const lc_bsa_plan_s *plan,
                                  const lc_rope3d_s *rope, int *dev_status, cudaStream_t stream,
                                  int *counter_scratch) {
  Sm100Params prm;
  memset(&prm, 0, sizeof(prm));
  const long long Nc = plan->Nc, Nn = plan->Nn, N = Nc + Nn;
  lc_status s = LC_OK;
  if (cached) {
    s = encode_segment(&prm.tmQ[1], q, batch, Nn, 0, Nn, heads);
    if (s == LC_OK) s = encode_segment(&prm.tmO[1], out, batch, Nn, 0, Nn, heads);
    if (s == LC_OK) s = encode_segment(&prm.tmK[1], k, batch, Nn, 0, Nn, heads);
    if (s == LC_OK) s = encode_segment(&prm.tmV[1], v, batch, Nn, 0, Nn, heads);
    if (s == LC_OK && Nc > 0) {
      s = encode_segment(&prm.tmK[0], cond_k, batch, Nc, 0, Nc, heads);
      if (s == LC_OK) s = encode_segment(&prm.tmV[0], cond_v, batch, Nc, 0, Nc, heads);
    }
    prm.q_row_offset_noisy = 0;
    prm.lse_nq = (int)Nn;
    prm.n_groups_active = plan->gn;
  } else {
    s = encode_segment(&prm.tmQ[1], q, batch, N, Nc, Nn, heads);
    if (s == LC_OK) s = encode_segment(&prm.tmO[1], out, batch, N, Nc, Nn, heads);
    if (s == LC_OK) s = encode_segment(&prm.tmK[1], k, batch, N, Nc, Nn, heads);
    if (s == LC_OK) s = encode_segment(&prm.tmV[1], v, batch, N, Nc, Nn, heads);
    if (s == LC_OK && Nc > 0) {
      s = encode_segment(&prm.tmQ[0], q, batch, N, 0, Nc, heads);
      if (s == LC_OK) s = encode_segment(&prm.tmO[0], out, batch, N, 0, Nc, heads);
      if (s == LC_OK) s = encode_segment(&prm.tmK[0], k, batch, N, 0, Nc, heads);
      if (s == LC_OK) s = encode_segment(&prm.tmV[0], v, batch, N, 0, Nc, heads);
    }
    prm.q_row_offset_noisy = (int)Nc;
    prm.lse_nq = (int)N;
    prm.n_groups_active = plan->G;
  }
  if (s != LC_OK) return s;
  if (Nc == 0) {  // keep the unused condition maps valid descriptors
    prm.tmQ[0] = prm.tmQ[1]; prm.tmK[0] = prm.tmK[1];
    prm.tmV[0] = prm.tmV[1]; prm.tmO[0] = prm.tmO[1];
  } else if (cached) {
    prm.tmQ[0] = prm.tmQ[1]; prm.tmO[0] = prm.tmO[1];
  }
  prm.rope_tab = rope->tab;
  prm.grp_ptr = plan->grp_ptr;
  prm.grp_ent = plan->grp_ent;
  prm.grp_order = plan->grp_order;
  prm.status = dev_status;
  prm.lse = lse;
  prm.timeout_ns = 2000000000LL;  // 2 s per wait
  prm.div_hw = lc_make_divmod(rope->H * rope->W);
  prm.div_w = lc_make_divmod(rope->W);
  prm.T = rope->T; prm.H = rope->H; prm.W = rope->W;
  prm.Nc = (int)Nc; prm.Nn = (int)Nn; prm.Cb = plan->Cb; prm.gc = plan->gc;
  prm.heads = heads;
  long long total = (long long)batch * heads * prm.n_groups_active;
  if (total == 0) return LC_OK;
  if (total >= (1LL << 31)) return LC_ERR_UNSUPPORTED;
  prm.total_items = (int)total;
  prm.tab_floats = (int)rope->n_floats;
  prm.scale_log2 = scale * 1.4426950408889634f;

  const size_t smem = 1024 + SmemOffsets::tab + sizeof(float) * (size_t)rope->n_floats;
  if (smem > 227 * 1024) return LC_ERR_UNSUPPORTED;
  LC_CUDA_TRY(cudaFuncSetAttribute(bsa_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)smem));
  int dev = 0, n_sm = 0;
  LC_CUDA_TRY(cudaGetDevice(&dev));
  LC_CUDA_TRY(cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev));
  const int grid = (int)(total < n_sm ? total : n_sm);

  if (counter_scratch) {  // caller-provided scratch: nothing is allocated
    prm.work_counter = counter_scratch;
    cudaError_t e = cudaMemsetAsync(counter_scratch, 0, sizeof(int), stream);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(stream, plan->ready, 0);
    if (e == cudaSuccess) {
      bsa_sm100_kernel<<<grid, kThreads, smem, stream>>>(prm);
      e = cudaGetLastError();
    }
    return lc_from_cuda(e);
  }
  int *counter = nullptr;
  LC_CUDA_TRY(cudaMallocAsync(&counter, sizeof(int), stream));
  prm.work_counter = counter;
  cudaError_t e = cudaMemsetAsync(counter, 0, sizeof(int), stream);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(stream, plan->ready, 0);
  if (e == cudaSuccess) {
    bsa_sm100_kernel<<<grid, kThreads, smem, stream>>>(prm);
    e = cudaGetLastError();
  }
  cudaError_t e2 = cudaFreeAsync(counter, stream);
  if (e == cudaSuccess) e = e2;
  return lc_from_cuda(e);
}

lc_status lc_launch_watchdog_selftest(int *dev_status, long long timeout_ns, cudaStream_t stream) {
  watchdog_selftest_kernel<<<1, 32, 0, stream>>>(dev_status, timeout_ns);
  LC_CUDA_TRY(cudaGetLastError());
  return LC_OK;
}
