// attn_bwd_sm100.cu -- tcgen05 backward of the block-sparse 3D-RoPE attention
// (bf16 inputs, fp32 accumulation): dk and dv written directly, dq summed in
// an fp32 buffer that attn_bwd.cu turns into dq.
//
// The gradients are the chain rule through the forward's definition (see
// attn_bwd.cu for the formulas and the pages that motivate them).  Layout of
// the work, one persistent CTA per SM:
//   work item = (batch, head, key group of up to 2 key blocks = 128 keys
//               with alike query lists), handed out longest query list
//               first; the group walks the sorted
//               union of the query blocks attending either key block (the
//               plan's key-group lists), two query blocks (128 queries) per
//               step.
//   per step, with keys as TMEM lanes (M = 128):
//     S^T  = K' Q'^T        dP^T = V dO^T          (tcgen05, into TMEM)
//     P^T  = exp(scale S^T - lse),  dS^T = P^T (scale dP^T - scale D)
//                           (warps 0-7, one key row and query block per
//                            thread; P^T written as bf16 pairs into TMEM 16
//                            queries at a time, dS^T held for the row until
//                            the previous step's dK / dQ are done, then
//                            written as bf16 tiles into shared memory, so the
//                            next step's S^T, dP^T can be computed while they
//                            are formed)
//     dV  += P^T dO         (A = P^T from TMEM, only dO read from shared memory)
//     dK' += dS^T Q'        (A from shared memory)
//     dQ'  = dS K'          (A = dS from shared memory, MN-major; queries as
//                            TMEM lanes), staged in shared memory by warps
//                            12-15 and added to the fp32 buffer by TMA
//                            reduce-adds
//   item end: dK = R^T dK' (and the RMSNorm transpose), dK and dV stored.
//   warp 8: TMA producer (K', V per item; Q', dO per step, 3 stages); warp 9:
//   MMA issuer; warps 10-11: stage log2e * lse and scale * D per step.
//   Q' = R(norm(q)) and K' = R(norm(k)) are formed once, before the kernel,
//   by the one-pass rotation the forward uses for K (same arithmetic).
//   TMEM: S^T [0,128) dP^T [128,256) dV [256,320) dK [320,384) dQ [384,448)
//         P^T [448,512).
// Every mbarrier wait is bounded; on expiry the CTA stops, drains and frees
// TMEM, and LC_DEVSTAT_TIMEOUT is set.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math.h>
#include <string.h>

#include "lc_internal.cuh"
#include "sm100_ptx.cuh"
#include "sm100_sync.cuh"

namespace {

using lcsm100::Ctx;
using lcsm100::drain_wait;
using lcsm100::wait_bar;
using lcsm100::wait_warp;

constexpr int kThreads = 512;
constexpr int kEwWarps = 8;       // 0-7: elementwise, two warps per key row (query halves)
constexpr int kWarpProducer = 8;
constexpr int kWarpMma = 9;
constexpr int kWarpRope = 10;     // and 11
constexpr int kRopeThreads = 64;
constexpr int kWarpDq = 12;       // 12-15
// Q' / dO stages: with three, a stage's reload is issued a whole step
// before the S^T / dP^T MMAs that read it (with two, the MMA issuer waited
// for the load after every step).
#ifndef LC_BWD_Q_STAGES
#define LC_BWD_Q_STAGES 3
#endif
constexpr int kQStages = LC_BWD_Q_STAGES;
constexpr int kTileBytes = 128 * 128;  // 128 rows x 64 bf16
constexpr int kBoxBytes = 64 * 128;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColST = 0, kColDPT = 128, kColDV = 256, kColDK = 320, kColDQ = 384;
constexpr uint32_t kColPT = 448;  // P^T as bf16 pairs (the A operand of dV)
constexpr uint32_t kIdescKQ = lcptx::idesc_bf16_f32(128, 128, 0, 0);  // S^T, dP^T
constexpr uint32_t kIdescAcc = lcptx::idesc_bf16_f32(128, 64, 0, 1);  // dV, dK (A K-major)
constexpr uint32_t kIdescDQ = lcptx::idesc_bf16_f32(128, 64, 1, 1);   // dQ (A = dS, MN-major)
constexpr float kLog2e = 1.4426950408889634f;
// Register split (setmaxnreg, per warpgroup): the two elementwise warpgroups
// hold two 32-column TMEM loads and their results; producer / MMA / RoPE need
// few; the dQ warpgroup holds one 64-column row.  The host refuses to launch
// unless the block's registers cover the split.
constexpr int kRegsEw = 160, kRegsCtl = 80, kRegsDq = 112;
constexpr int kRegsTotal = 256 * kRegsEw + 128 * (kRegsCtl + kRegsDq);
constexpr int kRegsAtLaunchMin = (kRegsTotal + kThreads - 1) / kThreads;
static_assert(kRegsTotal <= 65536, "register split");

struct __align__(64) BwdParams {
  CUtensorMap tmQ[2], tmK[2], tmV[2], tmG[2];  // [0] condition segment, [1] noisy; G = dO
  CUtensorMap tmDQ;                            // fp32 dq sums, half rows (reduce-add target)
  const float *rope_tab;
  const int *kg_ptr;
  const uint32_t *kg_ent;
  const int *kg_order;
  const int2 *kg_blk;
  int *work_counter;
  int *status;
  const float *lse;    // [B, heads, N] natural log (the forward's)
  const float *delta;  // [B, heads, N] rowsum(dO * O)
  float *dq_acc;       // [B, N, heads, 64] fp32, zero on entry
  float *dk_acc;       // [B, N, heads, 64] fp32 dk' (under an RMSNorm of k), or NULL
  __nv_bfloat16 *dk, *dv;
  long long timeout_ns;
  lc_divmod div_hw, div_w;
  int T, H, W;
  int Nc, Nn, Cb, kgc, heads, KG, total_items;
  int tab_floats;  // RoPE table floats copied to shared memory (0: read from global memory)
  int n_blocks;   // query / key blocks of the pattern (valid block ids: [0, n_blocks))
  int ent_cap;    // entries kg_ent holds (valid list bounds: [0, ent_cap])
  float scale;
};

struct SmemOffsets {
  static constexpr int k = 0;                                  // key tile K' (one item)
  static constexpr int v = k + kTileBytes;                     // value tile
  static constexpr int q = v + kTileBytes;                     // [kQStages] query tiles Q'
  static constexpr int g = q + kQStages * kTileBytes;          // [kQStages] dO tiles
  static constexpr int ds = g + kQStages * kTileBytes;         // dS^T, two 64-query tiles
  static constexpr int dq = ds + 2 * kTileBytes;               // dQ' staging: [block][half] 64 x 32 fp32
  static constexpr int lse = dq + 2 * kTileBytes;              // [kQStages][128] lse * log2e
  static constexpr int del = lse + kQStages * 128 * 4;         // [kQStages][128] scale * D
  static constexpr int bars = del + kQStages * 128 * 4;
  static constexpr int n_bars = 48;
  static constexpr int misc = bars + n_bars * 8;
  static constexpr int tab = misc + 64;  // the RoPE table, when it fits
};

enum {
  B_SCHED_FULL = 0,                 // [2]
  B_SCHED_EMPTY = 2,                // [2]
  B_KV_FULL = 4,                    // K', V landed
  B_KV_EMPTY = 5,                   // item's MMAs done with K', V
  B_ST_FREE = 6,                    // S^T, dP^T read out of TMEM (8 warps)
  B_QG_FULL = 8,                    // [kQStages] Q', dO landed
  B_QG_READY = B_QG_FULL + kQStages,   // lse / D staged
  B_QG_EMPTY = B_QG_READY + kQStages,  // step's MMAs done with Q, dO
  B_SDP = B_QG_EMPTY + kQStages,    // S^T and dP^T in TMEM
  B_PDS = B_SDP + 1,                // P^T in TMEM, dS^T in shared memory (8 warps)
  B_STEP = B_PDS + 1,               // step's dV, dK, dQ MMAs complete (dS^T tiles free)
  B_DQ_FULL = B_STEP + 1,           // dQ of a step in TMEM
  B_DQ_EMPTY = B_DQ_FULL + 1,       // dQ read out (4 warps)
  B_ACC = B_DQ_EMPTY + 1,           // item's dK, dV complete
  B_EPI_FREE = B_ACC + 1,           // dK, dV read out (8 warps)
  B_DQ_STAGED = B_EPI_FREE + 1,     // dQ' tile staged in shared memory (4 warps)
  B_DQ_SMEM_FREE = B_DQ_STAGED + 1, // its reduce-add has read the staging tile
  B_DRAIN = B_DQ_SMEM_FREE + 1,
  B_PT_FREE = B_DRAIN + 1,          // step's dV MMAs complete (P^T columns free)
  B_COUNT = B_PT_FREE + 1
};
static_assert(B_COUNT <= SmemOffsets::n_bars, "barrier space");
constexpr int kSchedConsumers = kEwWarps + 1 + 2 + 4;  // elementwise, MMA, RoPE, dQ warps

struct KItem {
  int b, h, seg, cnt, seg_len, len;
  int krow0, krow1;  // first row (in the segment) of each key block; past the end if absent
  __device__ int krow(int half) const { return half ? krow1 : krow0; }
  const uint32_t *ent;
};

// Device-side plan checks: a key group id, key block, list bound or query
// entry that a consistent plan never holds is replaced by a harmless one (a
// group with no valid key row, so nothing is stored; a one-entry list; an
// absent query block that loads as zeros, is masked and adds nothing to dq)
// before it is used as an index, a TMA coordinate or a store address, and
// LC_DEVSTAT_CHECK is raised by the role passed `status` (the producer).
__device__ __forceinline__ KItem decode_kitem(const BwdParams &p, int item, int *status) {
  KItem it;
  const int per = p.KG;
  const int bh = item / per;
  int g = p.kg_order[item - bh * per];
  bool bad = (unsigned)g >= (unsigned)p.KG;
  if (bad) g = 0;
  it.b = bh / p.heads;
  it.h = bh - it.b * p.heads;
  it.seg = g < p.kgc ? 0 : 1;
  int2 kb = p.kg_blk[g];  // global key block ids
  const int base = it.seg ? p.Cb : 0;
  const int nseg = it.seg ? p.n_blocks - p.Cb : p.Cb;  // key blocks of the segment
  it.seg_len = it.seg ? p.Nn : p.Nc;
  const bool x_ok = (unsigned)(kb.x - base) < (unsigned)nseg;
  const bool y_ok = kb.y < 0 || (unsigned)(kb.y - base) < (unsigned)nseg;
  if (!x_ok || !y_ok) {
    bad = true;
    it.cnt = 0;  // no key row of the item is valid: nothing is loaded or stored
    it.krow0 = it.krow1 = it.seg_len;
  } else {
    it.cnt = kb.y >= 0 ? 2 : 1;
    it.krow0 = 64 * (kb.x - base);
    it.krow1 = kb.y >= 0 ? 64 * (kb.y - base) : it.seg_len;
  }
  int lo = p.kg_ptr[g], hi = p.kg_ptr[g + 1];
  if (lo < 0 || hi <= lo || hi > p.ent_cap) {
    bad = true;
    lo = 0;
    hi = 1;
  }
  it.len = hi - lo;
  it.ent = p.kg_ent + lo;
  if (bad && status) atomicOr(status, LC_DEVSTAT_CHECK);
  return it;
}

// A list entry names a query block of the pattern and at least one member.
__device__ __forceinline__ bool qentry_ok(const BwdParams &p, uint32_t e) {
  return (int)(e & 0xFFFFFFu) < p.n_blocks && ((e >> 24) - 1u) < 3u;
}

// Query block of a list entry -> segment, first row in the segment, tokens.
__device__ __forceinline__ void qblock(const BwdParams &p, uint32_t e, int &seg, int &row,
                                       int &cnt) {
  const int r = (int)(e & 0xFFFFFFu);
  if (r < p.Cb) {
    seg = 0;
    row = 64 * r;
    cnt = min(64, p.Nc - row);
  } else {
    seg = 1;
    row = 64 * (r - p.Cb);
    cnt = min(64, p.Nn - row);
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

__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// cos / sin of pair p (0..31) at token n (the table in shared or global memory).
__device__ __forceinline__ void pair_angle(const BwdParams &a, const float *tab, int n, int p,
                                           float &c, float &s) {
  const int t = lc_div(n, a.div_hw);
  const int rem = n - t * a.div_hw.d;
  const int hh = lc_div(rem, a.div_w);
  const int w = rem - hh * a.div_w.d;
  if (p < 8) {
    c = tab[t * 8 + p];
    s = tab[a.T * 8 + t * 8 + p];
  } else if (p < 20) {
    c = tab[a.T * 16 + hh * 12 + p - 8];
    s = tab[a.T * 16 + a.H * 12 + hh * 12 + p - 8];
  } else {
    c = tab[a.T * 16 + a.H * 24 + w * 12 + p - 20];
    s = tab[a.T * 16 + a.H * 24 + a.W * 12 + w * 12 + p - 20];
  }
}

// kNorm: k is RMS-normalised, so dK' goes out in fp32 for the finalize pass
// (the plain path is a separate instantiation without that branch).
template <bool kNorm>
__global__ void __launch_bounds__(kThreads, 1) bsa_bwd_sm100_kernel(const __grid_constant__ BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  uint8_t *sK = smem + SmemOffsets::k;
  uint8_t *sV = smem + SmemOffsets::v;
  uint8_t *sQ = smem + SmemOffsets::q;
  uint8_t *sG = smem + SmemOffsets::g;
  uint8_t *sDS = smem + SmemOffsets::ds;
  float *sLse = reinterpret_cast<float *>(smem + SmemOffsets::lse);
  float *sDel = reinterpret_cast<float *>(smem + SmemOffsets::del);
  uint32_t *misc = reinterpret_cast<uint32_t *>(smem + SmemOffsets::misc);
  // misc[0] tmem base, misc[1..2] scheduled items, misc[3] abort flag
  float *stab = reinterpret_cast<float *>(smem + SmemOffsets::tab);
  const float *tab = p.tab_floats ? stab : p.rope_tab;
  Ctx ctx;
  ctx.bar0 = lcptx::smem_addr(smem + SmemOffsets::bars);
  ctx.abort_flag = reinterpret_cast<volatile int *>(&misc[3]);
  ctx.status = p.status;
  ctx.timeout_ns = p.timeout_ns;
  const long long N = (long long)p.Nc + p.Nn;

  for (int i = tid; i < p.tab_floats; i += kThreads) stab[i] = p.rope_tab[i];
  if (tid == 0) {
    misc[3] = 0;
    for (int i = 0; i < 2; ++i) {
      lcptx::mbar_init(ctx.bar(B_SCHED_FULL + i), 1);
      lcptx::mbar_init(ctx.bar(B_SCHED_EMPTY + i), kSchedConsumers);
    }
    lcptx::mbar_init(ctx.bar(B_KV_FULL), 1);
    lcptx::mbar_init(ctx.bar(B_KV_EMPTY), 1);
    lcptx::mbar_init(ctx.bar(B_ST_FREE), kEwWarps);
    for (int s = 0; s < kQStages; ++s) {
      lcptx::mbar_init(ctx.bar(B_QG_FULL + s), 1);
      lcptx::mbar_init(ctx.bar(B_QG_READY + s), kRopeThreads);
      lcptx::mbar_init(ctx.bar(B_QG_EMPTY + s), 1);
    }
    lcptx::mbar_init(ctx.bar(B_SDP), 1);
    lcptx::mbar_init(ctx.bar(B_PDS), kEwWarps);
    lcptx::mbar_init(ctx.bar(B_STEP), 1);
    lcptx::mbar_init(ctx.bar(B_PT_FREE), 1);
    lcptx::mbar_init(ctx.bar(B_DQ_FULL), 1);
    lcptx::mbar_init(ctx.bar(B_DQ_EMPTY), 4);
    lcptx::mbar_init(ctx.bar(B_ACC), 1);
    lcptx::mbar_init(ctx.bar(B_EPI_FREE), kEwWarps);
    lcptx::mbar_init(ctx.bar(B_DQ_STAGED), 4);
    lcptx::mbar_init(ctx.bar(B_DQ_SMEM_FREE), 1);
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
      lcptx::tma_prefetch_desc(&p.tmG[i]);
    }
    lcptx::tma_prefetch_desc(&p.tmDQ);
  }
  lcptx::tc_fence_before();
  __syncthreads();
  lcptx::tc_fence_after();
  const uint32_t tmem = misc[0];

  if (warp >= kWarpProducer && warp < kWarpDq) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsCtl));
  if (warp == kWarpProducer) {
    // ======================= TMA producer (one thread) =======================
    if (lane == 0) {
      uint32_t item_it = 0, q_it = 0;
      uint32_t kv_valid = 0, kv_par = 0, q_valid = 0, q_par = 0;  // for the drain
      for (;;) {
        const int slot = item_it & 1;
        int item = atomicAdd(p.work_counter, 1);
        if (item >= p.total_items) item = -1;
        if (!wait_bar(ctx, ctx.bar(B_SCHED_EMPTY + slot), ((item_it >> 1) & 1) ^ 1)) break;
        misc[1 + slot] = (uint32_t)item;
        lcptx::mbar_arrive(ctx.bar(B_SCHED_FULL + slot));
        if (item < 0) break;
        const KItem it = decode_kitem(p, item, p.status);
        const uint32_t kph = item_it & 1;
        bool ok = wait_bar(ctx, ctx.bar(B_KV_EMPTY), kph ^ 1);
        if (!ok) break;
        {
          const uint32_t bar = ctx.bar(B_KV_FULL);
          lcptx::mbar_arrive_expect_tx(bar, 2 * kTileBytes);
          const uint32_t dk = lcptx::smem_addr(sK);
          const uint32_t dv = lcptx::smem_addr(sV);
          // rows past the segment end (a missing second block) read as zeros
          lcptx::tma_load_4d(dk, &p.tmK[it.seg], bar, 0, it.h, it.krow0, it.b);
          lcptx::tma_load_4d(dk + kBoxBytes, &p.tmK[it.seg], bar, 0, it.h, it.krow1, it.b);
          lcptx::tma_load_4d(dv, &p.tmV[it.seg], bar, 0, it.h, it.krow0, it.b);
          lcptx::tma_load_4d(dv + kBoxBytes, &p.tmV[it.seg], bar, 0, it.h, it.krow1, it.b);
          kv_valid = 1u;
          kv_par = kph;
        }
        const int nsteps = (it.len + 1) >> 1;
        for (int t = 0; t < nsteps && ok; ++t, ++q_it) {
          const int s = q_it % kQStages;
          const uint32_t ph = (q_it / kQStages) & 1;
          ok = wait_bar(ctx, ctx.bar(B_QG_EMPTY + s), ph ^ 1);
          if (!ok) break;
          // (TMA loads may start anywhere: an entry that fails the plan check
          // reads zeros or other rows here; the dQ and lse / D paths, which
          // address memory with it, check it and report it)
          int sa, ra, na, sb, rb, nb;
          qblock(p, __ldg(it.ent + 2 * t), sa, ra, na);
          if (2 * t + 1 < it.len) {
            qblock(p, __ldg(it.ent + 2 * t + 1), sb, rb, nb);
          } else {  // no second query block: a box past the noisy segment's end reads zeros
            sb = 1;
            rb = p.Nn;
          }
          const uint32_t bar = ctx.bar(B_QG_FULL + s);
          lcptx::mbar_arrive_expect_tx(bar, 2 * kTileBytes);
          const uint32_t dq = lcptx::smem_addr(sQ + s * kTileBytes);
          const uint32_t dg = lcptx::smem_addr(sG + s * kTileBytes);
          lcptx::tma_load_4d(dq, &p.tmQ[sa], bar, 0, it.h, ra, it.b);
          lcptx::tma_load_4d(dq + kBoxBytes, &p.tmQ[sb], bar, 0, it.h, rb, it.b);
          lcptx::tma_load_4d(dg, &p.tmG[sa], bar, 0, it.h, ra, it.b);
          lcptx::tma_load_4d(dg + kBoxBytes, &p.tmG[sb], bar, 0, it.h, rb, it.b);
          q_valid |= 1u << s;
          q_par = (q_par & ~(1u << s)) | (ph << s);
        }
        if (!ok) break;
        ++item_it;
      }
      // Drain: every load this thread issued must land before the CTA exits.
      if (kv_valid) drain_wait(ctx.bar(B_KV_FULL), kv_par, p.timeout_ns);
      for (int s = 0; s < kQStages; ++s)
        if ((q_valid >> s) & 1u) drain_wait(ctx.bar(B_QG_FULL + s), (q_par >> s) & 1u, p.timeout_ns);
    }
  } else if (warp == kWarpMma) {
    // ======================= MMA issuer (one thread) =========================
    if (lane == 0) {
      uint32_t item_it = 0, q_it = 0, k_step = 0;
      uint32_t pds_ph = 0;
      constexpr uint32_t kDescHi = (1024u >> 4) | (1u << 14) | (2u << 29);
      constexpr uint32_t kTileLo = kTileBytes >> 4;
      auto desc = [](uint32_t lo) -> uint64_t {
        return (static_cast<uint64_t>(kDescHi) << 32) | lo;
      };
      // K-major operands (leading byte offset 16) and MN-major ones with one
      // 64-element chunk (leading byte offset unused); dS^T as the MN-major A
      // of dQ has two 64-query chunks 16 KB apart.
      const uint32_t k_km = (lcptx::smem_addr(sK) >> 4) | (1u << 16);
      const uint32_t v_km = (lcptx::smem_addr(sV) >> 4) | (1u << 16);
      const uint32_t q_km = (lcptx::smem_addr(sQ) >> 4) | (1u << 16);
      const uint32_t g_km = (lcptx::smem_addr(sG) >> 4) | (1u << 16);
      const uint32_t k_mn = (lcptx::smem_addr(sK) >> 4) | (512u << 16);
      const uint32_t q_mn = (lcptx::smem_addr(sQ) >> 4) | (512u << 16);
      const uint32_t g_mn = (lcptx::smem_addr(sG) >> 4) | (512u << 16);
      const uint32_t ds_mn = (lcptx::smem_addr(sDS) >> 4) | ((uint32_t)(kTileBytes >> 4) << 16);
      const uint32_t ds_km = (lcptx::smem_addr(sDS) >> 4) | (1u << 16);
      uint32_t st_free_ph = 0;
      // S^T = K' Q'^T and dP^T = V dO^T of step q (stage s) into TMEM, once the
      // previous step's S^T / dP^T have been read out.
      auto issue_sdp = [&](int s, uint32_t ph, bool wait_free) -> bool {
        if (!wait_bar(ctx, ctx.bar(B_QG_FULL + s), ph)) return false;
        if (wait_free) {
          if (!wait_bar(ctx, ctx.bar(B_ST_FREE), st_free_ph)) return false;
          st_free_ph ^= 1;
        }
        lcptx::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          lcptx::mma_ss(tmem + kColST, desc(k_km + 2 * kk), desc(q_km + s * kTileLo + 2 * kk),
                        kIdescKQ, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          lcptx::mma_ss(tmem + kColDPT, desc(v_km + 2 * kk), desc(g_km + s * kTileLo + 2 * kk),
                        kIdescKQ, kk > 0);
        lcptx::mma_commit(ctx.bar(B_SDP));
        return true;
      };
      for (;;) {
        const int slot = item_it & 1;
        if (!wait_bar(ctx, ctx.bar(B_SCHED_FULL + slot), (item_it >> 1) & 1)) break;
        const int item = (int)misc[1 + slot];
        lcptx::mbar_arrive(ctx.bar(B_SCHED_EMPTY + slot));
        if (item < 0) break;
        const KItem it = decode_kitem(p, item, nullptr);
        bool ok = wait_bar(ctx, ctx.bar(B_KV_FULL), item_it & 1);
        const int nsteps = (it.len + 1) >> 1;
        if (ok) ok = issue_sdp(q_it % kQStages, (q_it / kQStages) & 1, k_step > 0);
        for (int t = 0; t < nsteps && ok; ++t, ++q_it, ++k_step) {
          const int s = q_it % kQStages;
          // the next step's S^T / dP^T overlap this step's elementwise pass
          if (t + 1 < nsteps) {
            ok = issue_sdp((q_it + 1) % kQStages, ((q_it + 1) / kQStages) & 1, true);
            if (!ok) break;
          }
          ok = wait_bar(ctx, ctx.bar(B_PDS), pds_ph);
          if (!ok) break;
          pds_ph ^= 1;
          if (t == 0 && item_it > 0) {  // the previous item's dK, dV have been read out
            ok = wait_bar(ctx, ctx.bar(B_EPI_FREE), (item_it - 1) & 1);
            if (!ok) break;
          }
          lcptx::tc_fence_after();
          // dV += P^T dO with P^T in TMEM (only dO is read from shared memory);
          // dK' += dS^T Q' with dS^T from the 64-query tiles in shared memory
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            lcptx::mma_ts(tmem + kColDV, tmem + kColPT + 8 * kk,
                          desc(g_mn + s * kTileLo + 128 * kk), kIdescAcc, (t > 0 || kk > 0) ? 1u : 0u);
          lcptx::mma_commit(ctx.bar(B_PT_FREE));
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            lcptx::mma_ss(tmem + kColDK, desc(ds_km + (kk >> 2) * kTileLo + 2 * (kk & 3)),
                          desc(q_mn + s * kTileLo + 128 * kk), kIdescAcc, (t > 0 || kk > 0) ? 1u : 0u);
          if (k_step > 0) {  // the dQ warps have read the previous step's dQ
            ok = wait_bar(ctx, ctx.bar(B_DQ_EMPTY), (k_step - 1) & 1);
            if (!ok) break;
            lcptx::tc_fence_after();
          }
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            lcptx::mma_ss(tmem + kColDQ, desc(ds_mn + 128 * kk), desc(k_mn + 128 * kk), kIdescDQ,
                          kk > 0);
          lcptx::mma_commit(ctx.bar(B_DQ_FULL));
          lcptx::mma_commit(ctx.bar(B_QG_EMPTY + s));
          lcptx::mma_commit(ctx.bar(B_STEP));
          if (t + 1 == nsteps) {
            lcptx::mma_commit(ctx.bar(B_ACC));
            lcptx::mma_commit(ctx.bar(B_KV_EMPTY));
          }
        }
        if (!ok) break;
        ++item_it;
      }
      lcptx::mma_commit(ctx.bar(B_DRAIN));
      drain_wait(ctx.bar(B_DRAIN), 0, p.timeout_ns);
    }
    __syncwarp();
  } else {
    // ======================= warps 10-11: stage lse / D per step =============
    const int rt = tid - kWarpRope * 32;
    uint32_t item_it = 0, q_it = 0;
    for (;;) {
      const int slot = item_it & 1;
      if (!wait_warp(ctx, ctx.bar(B_SCHED_FULL + slot), (item_it >> 1) & 1)) break;
      const int item = (int)misc[1 + slot];
      __syncwarp();
      if (lane == 0) lcptx::mbar_arrive(ctx.bar(B_SCHED_EMPTY + slot));
      if (item < 0) break;
      const KItem it = decode_kitem(p, item, nullptr);
      bool ok = true;
      const int nsteps = (it.len + 1) >> 1;
      const float *lse_bh = p.lse + ((long long)it.b * p.heads + it.h) * N;
      const float *del_bh = p.delta + ((long long)it.b * p.heads + it.h) * N;
      for (int t = 0; t < nsteps && ok; ++t, ++q_it) {
        const int s = q_it % kQStages;
        // This thread's two query rows (rt of each query block): log2e * lse
        // and scale * D of their tokens.  A row that does not exist (past a
        // block's last token, an absent block, an entry failing the plan
        // check) gets lse = +inf, so its P is exactly 0 in every key row.
        float l2r[2], dlr[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          l2r[i] = __int_as_float(0x7f800000);
          dlr[i] = 0.f;
          const int e = 2 * t + i;
          if (e < it.len && qentry_ok(p, __ldg(it.ent + e))) {
            int qs, qr, qn;
            qblock(p, __ldg(it.ent + e), qs, qr, qn);
            if (rt < qn) {
              const int tok = (qs ? p.Nc : 0) + qr + rt;
              l2r[i] = __ldg(lse_bh + tok) * kLog2e;
              dlr[i] = __ldg(del_bh + tok) * p.scale;
            }
          }
        }
        // the stage is free once its previous step's MMAs are done, which the
        // producer's reload of it implies
        ok = wait_warp(ctx, ctx.bar(B_QG_FULL + s), (q_it / kQStages) & 1);
        if (!ok) break;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          sLse[s * 128 + rt + 64 * i] = l2r[i];
          sDel[s * 128 + rt + 64 * i] = dlr[i];
        }
        lcptx::mbar_arrive(ctx.bar(B_QG_READY + s));
      }
      if (!ok) break;
      ++item_it;
    }
  }
  } else if (warp >= kWarpDq) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsDq));
    // ======================= dQ warps: TMEM dQ' -> shared -> TMA reduce-add ==
    // Each step's dQ' tile (128 query rows x 64 fp32) is staged in shared
    // memory as four 64-row x 32-channel swizzled boxes and added into the
    // fp32 dq sums by the TMA engine (one thread issues; nothing per lane
    // goes to global memory).  Rows of absent or padded queries are zero.
    const int qrow = tid - kWarpDq * 32;  // TMEM lane == query row of the step
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    uint8_t *sDQ = smem + SmemOffsets::dq;
    uint32_t item_it = 0, dq_ph = 0, dq_step = 0;
    bool issued = false;
    for (;;) {
      const int slot = item_it & 1;
      if (!wait_warp(ctx, ctx.bar(B_SCHED_FULL + slot), (item_it >> 1) & 1)) break;
      const int item = (int)misc[1 + slot];
      __syncwarp();
      if (lane == 0) lcptx::mbar_arrive(ctx.bar(B_SCHED_EMPTY + slot));
      if (item < 0) break;
      const KItem it = decode_kitem(p, item, nullptr);
      const int nsteps = (it.len + 1) >> 1;
      bool ok = true;
      for (int t = 0; t < nsteps; ++t, ++dq_step) {
        // the step's two list entries (reduce-add coordinates), loaded while
        // the step's dQ is computed
        uint32_t ents[2] = {0u, 0u};
        if (qrow == 0) {
#pragma unroll
          for (int blk = 0; blk < 2; ++blk)
            if (2 * t + blk < it.len) ents[blk] = __ldg(it.ent + 2 * t + blk);
        }
        ok = wait_warp(ctx, ctx.bar(B_DQ_FULL), dq_ph);
        if (!ok) break;
        dq_ph ^= 1;
        lcptx::tc_fence_after();
        uint32_t a[2][32];
        lcptx::tmem_ld32(tmem + lane_base + kColDQ, a[0]);
        lcptx::tmem_ld32(tmem + lane_base + kColDQ + 32, a[1]);
        lcptx::tmem_wait_ld();
        lcptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) lcptx::mbar_arrive(ctx.bar(B_DQ_EMPTY));
        // the previous step's reduce-add has finished reading the staging tile
        ok = wait_warp(ctx, ctx.bar(B_DQ_SMEM_FREE), (dq_step & 1) ^ 1);
        if (!ok) break;
#pragma unroll
        for (int hd = 0; hd < 2; ++hd) {
          uint8_t *tile = sDQ + ((qrow >> 6) * 2 + hd) * (64 * 128);
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4 *>(tile + swz(qrow & 63, c)) =
                make_uint4(a[hd][4 * c], a[hd][4 * c + 1], a[hd][4 * c + 2], a[hd][4 * c + 3]);
        }
        lcptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) lcptx::mbar_arrive(ctx.bar(B_DQ_STAGED));
        if (qrow == 0) {
          ok = wait_bar(ctx, ctx.bar(B_DQ_STAGED), dq_step & 1);
          if (ok) {
#pragma unroll
            for (int blk = 0; blk < 2; ++blk) {
              const int e = 2 * t + blk;
              if (e >= it.len) continue;
              const uint32_t ent = ents[blk];
              if (!qentry_ok(p, ent)) {
                atomicOr(p.status, LC_DEVSTAT_CHECK);
                continue;
              }
              int qs, qr, qn;
              qblock(p, ent, qs, qr, qn);
              const int tok0 = (qs ? p.Nc : 0) + qr;
#pragma unroll
              for (int hd = 0; hd < 2; ++hd)
                lcptx::tma_reduce_add_4d(&p.tmDQ,
                                         lcptx::smem_addr(sDQ + (blk * 2 + hd) * (64 * 128)),
                                         32 * hd, it.h, tok0, it.b);
            }
            lcptx::bulk_commit_group();
            issued = true;
            lcptx::bulk_wait_group_read0();
            lcptx::mbar_arrive(ctx.bar(B_DQ_SMEM_FREE));
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0 && !*ctx.abort_flag;
        if (!ok) break;
      }
      if (!ok) break;
      ++item_it;
    }
    if (qrow == 0 && issued) lcptx::bulk_wait_group0();  // every reduce-add complete
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsEw));
    // ======================= elementwise warps 0-7 ===========================
    // Thread = key row kr (TMEM lane); warps 0-3 take the step's first query
    // block (columns 0-63), warps 4-7 the second: two warps per sub-partition
    // keep the exp unit busy.
    const int kr = tid & 127;
    const int half = warp >> 2;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tST = tmem + lane_base + kColST, tDPT = tmem + lane_base + kColDPT;
    const float sl2 = p.scale * kLog2e;
    const float2 sl2x2 = make_float2(sl2, sl2), scx2 = make_float2(p.scale, p.scale);
    uint32_t item_it = 0, q_it = 0, sdp_ph = 0;
    for (;;) {
      const int slot = item_it & 1;
      if (!wait_warp(ctx, ctx.bar(B_SCHED_FULL + slot), (item_it >> 1) & 1)) break;
      const int item = (int)misc[1 + slot];
      __syncwarp();
      if (lane == 0) lcptx::mbar_arrive(ctx.bar(B_SCHED_EMPTY + slot));
      if (item < 0) break;
      const KItem it = decode_kitem(p, item, nullptr);
      const bool key_valid = (kr >> 6) < it.cnt && it.krow(kr >> 6) + (kr & 63) < it.seg_len;
      const int nsteps = (it.len + 1) >> 1;
      bool ok = true;
      // This warp's list entry for the step: fetched one step ahead, so the
      // load's latency hides behind the previous step (0 = no query block).
      uint32_t ent_next = half < it.len ? __ldg(it.ent + half) : 0u;
      for (int t = 0; t < nsteps; ++t, ++q_it) {
        const int s = q_it % kQStages;
        const uint32_t ent = ent_next;
        const int e_next = 2 * (t + 1) + half;
        ent_next = e_next < it.len ? __ldg(it.ent + e_next) : 0u;
        // Does this warp's key block attend the step's query block?  The same
        // answer for all the warp's rows (one key block, one list entry), so
        // the branch below is uniform.  Within an attending block every pair
        // is attended: the query tokens a block lacks have lse = +inf; key
        // rows past a segment's end meet zero K' / V rows (their P, clamped
        // at 1, reaches no stored gradient).
        const bool member = ((ent >> (24 + (kr >> 6))) & 1u) != 0;
        // the staged lse / D of this step (written by the RoPE warps), then S^T, dP^T
        ok = wait_warp(ctx, ctx.bar(B_QG_READY + s), (q_it / kQStages) & 1) &&
             wait_warp(ctx, ctx.bar(B_SDP), sdp_ph);
        if (!ok) break;
        sdp_ph ^= 1;
        lcptx::tc_fence_after();
        const float *l2 = sLse + s * 128, *dl = sDel + s * 128;
        uint8_t *tile = sDS + half * kTileBytes;  // dS^T, this query block's MN-major chunk
        // P^T goes to TMEM chunk by chunk (after the wait for the previous
        // step's dV, which lands during the first chunk); dS^T of the whole
        // row is held, packed, until the previous step's dK / dQ are done
        // with the tile
        uint32_t dk[4][8];
        if (member) {
          // 16 queries at a time; the next chunk's TMEM loads are in flight
          // while this one is computed (double buffer)
          uint32_t sr[2][16], dr[2][16];
          lcptx::tmem_ld16(tST + 64 * half, sr[0]);
          lcptx::tmem_ld16(tDPT + 64 * half, dr[0]);
          lcptx::tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int c = 4 * half + k;
            if (k < 3) {
              lcptx::tmem_ld16(tST + 64 * half + 16 * (k + 1), sr[(k + 1) & 1]);
              lcptx::tmem_ld16(tDPT + 64 * half + 16 * (k + 1), dr[(k + 1) & 1]);
            } else {  // every TMEM load of the step has landed: S^T, dP^T may be overwritten
              lcptx::tc_fence_before();
              __syncwarp();
              if (lane == 0) lcptx::mbar_arrive(ctx.bar(B_ST_FREE));
            }
            const uint32_t(&scur)[16] = sr[k & 1];
            const uint32_t(&dcur)[16] = dr[k & 1];
            uint32_t pk[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              // log2e * lse and scale * D of queries 2i, 2i + 1 of the chunk
              // (16-byte shared loads, one per four queries)
              const float4 l4 = reinterpret_cast<const float4 *>(l2 + 16 * c)[i >> 1];
              const float4 d4 = reinterpret_cast<const float4 *>(dl + 16 * c)[i >> 1];
              const float2 nlq = (i & 1) ? make_float2(-l4.z, -l4.w) : make_float2(-l4.x, -l4.y);
              const float2 ndq = (i & 1) ? make_float2(-d4.z, -d4.w) : make_float2(-d4.x, -d4.y);
              // P = 2^(log2e (scale S - lse)) <= 1; dS = P * (scale dP - scale D),
              // two queries per packed fp32 instruction
              const float2 x = __ffma2_rn(
                  make_float2(__uint_as_float(scur[2 * i]), __uint_as_float(scur[2 * i + 1])), sl2x2, nlq);
              const float2 pv = make_float2(ex2(fminf(x.x, 0.f)), ex2(fminf(x.y, 0.f)));
              const float2 g = __ffma2_rn(
                  make_float2(__uint_as_float(dcur[2 * i]), __uint_as_float(dcur[2 * i + 1])), scx2, ndq);
              const float2 dv2 = __fmul2_rn(pv, g);
              pk[i] = pack_bf16(pv.x, pv.y);
              dk[k][i] = pack_bf16(dv2.x, dv2.y);
            }
            if (k == 0 && q_it > 0) {  // the previous step's dV is done with the P^T columns
              ok = wait_warp(ctx, ctx.bar(B_PT_FREE), (q_it - 1) & 1);
              lcptx::tc_fence_after();
            }
            // P^T row kr, this block's queries 16k .. 16k + 15: TMEM columns 32 * half + 8k ..
            if (ok) lcptx::tmem_st8(tmem + lane_base + kColPT + 32 * half + 8 * k, pk);
            if (k < 3) lcptx::tmem_wait_ld();
          }
        } else {
          // no pair of this key block and query block is attended: P^T and
          // dS^T are zero, and S^T / dP^T need not be read
          lcptx::tc_fence_before();
          __syncwarp();
          if (lane == 0) lcptx::mbar_arrive(ctx.bar(B_ST_FREE));
          if (q_it > 0) {
            ok = wait_warp(ctx, ctx.bar(B_PT_FREE), (q_it - 1) & 1);
            lcptx::tc_fence_after();
          }
          const uint32_t zero[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            if (ok) lcptx::tmem_st8(tmem + lane_base + kColPT + 32 * half + 8 * k, zero);
#pragma unroll
            for (int i = 0; i < 8; ++i) dk[k][i] = 0u;
          }
        }
        if (!ok) {
          lcptx::tmem_wait_st();
          break;
        }
        if (q_it > 0) {  // the previous step's dK / dQ are done with the dS^T tiles
          ok = wait_warp(ctx, ctx.bar(B_STEP), (q_it - 1) & 1);
          if (!ok) {
            lcptx::tmem_wait_st();
            break;
          }
        }
        // row kr of the dS^T tile: 64 queries of this block, 128-byte swizzled;
        // K-major for dK, MN-major (dS) for dQ
#pragma unroll
        for (int k = 0; k < 4; ++k) {
#pragma unroll
          for (int i = 0; i < 2; ++i)
            *reinterpret_cast<uint4 *>(tile + swz(kr, k * 2 + i)) =
                make_uint4(dk[k][4 * i], dk[k][4 * i + 1], dk[k][4 * i + 2], dk[k][4 * i + 3]);
        }
        lcptx::tmem_wait_st();
        lcptx::tc_fence_before();
        lcptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) lcptx::mbar_arrive(ctx.bar(B_PDS));
      }
      if (!ok) break;
      // ---- epilogue: warps 0-3 store dV; warps 4-7 store dK = R^T dK' as bf16
      // rows straight to global memory, or, when k is normalised, dK' in fp32
      // for the finalize pass (R^T and the RMSNorm transpose).
      ok = wait_warp(ctx, ctx.bar(B_ACC), item_it & 1);
      if (!ok) break;
      lcptx::tc_fence_after();
      const int tok = (it.seg ? p.Nc : 0) + it.krow(kr >> 6) + (kr & 63);
      const long long off = (((long long)it.b * N + tok) * p.heads + it.h) * LC_HEAD_DIM;
      float acc[64];
      {
        uint32_t a[32], b2[32];
        const uint32_t col = half ? kColDK : kColDV;
        lcptx::tmem_ld32(tmem + lane_base + col, a);
        lcptx::tmem_ld32(tmem + lane_base + col + 32, b2);
        lcptx::tmem_wait_ld();
#pragma unroll
        for (int d = 0; d < 32; ++d) {
          acc[d] = __uint_as_float(a[d]);
          acc[32 + d] = __uint_as_float(b2[d]);
        }
      }
      lcptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) lcptx::mbar_arrive(ctx.bar(B_EPI_FREE));
      if (key_valid) {
        if (kNorm && half && p.dk_acc) {  // dk' as is; R^T and the norm transpose follow
          float4 *dst = reinterpret_cast<float4 *>(p.dk_acc + off);
#pragma unroll
          for (int c = 0; c < 16; ++c)
            dst[c] = make_float4(acc[4 * c], acc[4 * c + 1], acc[4 * c + 2], acc[4 * c + 3]);
        } else {
          if (half) {
#pragma unroll
            for (int q2 = 0; q2 < 32; ++q2) {  // R^T: turn each pair back
              float c, sn;
              pair_angle(p, tab, tok, q2, c, sn);
              const float u = acc[2 * q2], w = acc[2 * q2 + 1];
              acc[2 * q2] = fmaf(u, c, w * sn);
              acc[2 * q2 + 1] = fmaf(w, c, -u * sn);
            }
          }
          uint4 *dst = reinterpret_cast<uint4 *>((half ? p.dk : p.dv) + off);
#pragma unroll
          for (int c = 0; c < 8; ++c)
            dst[c] = make_uint4(pack_bf16(acc[8 * c], acc[8 * c + 1]),
                                pack_bf16(acc[8 * c + 2], acc[8 * c + 3]),
                                pack_bf16(acc[8 * c + 4], acc[8 * c + 5]),
                                pack_bf16(acc[8 * c + 6], acc[8 * c + 7]));
        }
      }
      ++item_it;
    }
  }

  // ---- teardown
  lcptx::tc_fence_before();
  __syncthreads();
  lcptx::tc_fence_after();
  if (warp == kWarpMma) lcptx::tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

lc_status lc_launch_backward_sm100(const void *q, const void *k, const void *v, const void *out,
                                   const float *lse, const void *dout, void *dq, void *dk,
                                   void *dv, int batch, int heads, float scale,
                                   const lc_qk_norm &norm, const lc_bsa_plan_s *plan,
                                   const lc_rope3d_s *rope, cudaStream_t stream) {
  BwdParams prm;
  memset(&prm, 0, sizeof(prm));
  const long long Nc = plan->Nc, Nn = plan->Nn, N = Nc + Nn;
  const long long total = (long long)batch * heads * plan->KG;
  if (total == 0) return LC_OK;
  if (total >= (1LL << 31)) return LC_ERR_UNSUPPORTED;
  // the RoPE table goes to shared memory when it fits beside the tiles
  static_assert(1024 + SmemOffsets::tab <= 227 * 1024, "shared memory");
  const size_t tab_bytes = sizeof(float) * (size_t)rope->n_floats;
  const bool tab_in_smem = 1024 + SmemOffsets::tab + tab_bytes <= 227 * 1024;
  const size_t smem = 1024 + SmemOffsets::tab + (tab_in_smem ? tab_bytes : 0);
  lc_status s = LC_OK;
  prm.status = lc_device_status_ptr(&s);
  if (s != LC_OK) return s;
  cudaMemPool_t pool = lc_scratch_pool(&s);
  if (s != LC_OK) return s;
  const bool with_norm = norm.k_w != nullptr;
  void (*const kern)(const BwdParams) = with_norm ? bsa_bwd_sm100_kernel<true>
                                                  : bsa_bwd_sm100_kernel<false>;
  static int regs_at_launch[2] = {-1, -1};
  int &regs = regs_at_launch[with_norm ? 1 : 0];
  if (regs < 0) {
    cudaFuncAttributes fa;
    LC_CUDA_TRY(cudaFuncGetAttributes(&fa, kern));
    regs = fa.numRegs;
  }
  if (regs < kRegsAtLaunchMin) return LC_ERR_UNSUPPORTED;  // the split could never complete
  LC_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  int dev = 0, n_sm = 0;
  LC_CUDA_TRY(cudaGetDevice(&dev));
  LC_CUDA_TRY(cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev));
  LC_CUDA_TRY(cudaStreamWaitEvent(stream, plan->ready, 0));
  LC_CUDA_TRY(cudaStreamWaitEvent(stream, rope->ready, 0));

  // Scratch from the library's pool: D, the fp32 dq sums, the scheduler
  // counter, and Q' = R(norm(q)), K' = R(norm(k)).
  const size_t rows = (size_t)batch * N * heads;
  const size_t tbytes = rows * LC_HEAD_DIM * 2;
  float *delta = nullptr, *dq_acc = nullptr, *dk_acc = nullptr;
  int *counter = nullptr;
  void *q_rot = nullptr, *k_rot = nullptr;
  cudaError_t e = cudaMallocFromPoolAsync(reinterpret_cast<void **>(&delta), rows * sizeof(float),
                                          pool, stream);
  if (e == cudaSuccess)
    e = cudaMallocFromPoolAsync(reinterpret_cast<void **>(&dq_acc),
                                rows * LC_HEAD_DIM * sizeof(float), pool, stream);
  if (e == cudaSuccess)
    e = cudaMallocFromPoolAsync(reinterpret_cast<void **>(&counter), sizeof(int), pool, stream);
  if (e == cudaSuccess) e = cudaMallocFromPoolAsync(&q_rot, tbytes, pool, stream);
  if (e == cudaSuccess) e = cudaMallocFromPoolAsync(&k_rot, tbytes, pool, stream);
  if (e == cudaSuccess && norm.k_w)  // dk' in fp32, normalised back by the finalize pass
    e = cudaMallocFromPoolAsync(reinterpret_cast<void **>(&dk_acc),
                                rows * LC_HEAD_DIM * sizeof(float), pool, stream);
  if (e == cudaSuccess)
    e = cudaMemsetAsync(dq_acc, 0, rows * LC_HEAD_DIM * sizeof(float), stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(counter, 0, sizeof(int), stream);
  if (e == cudaSuccess) s = lc_rope_rows_bf16(q, q_rot, batch, N, heads, 0, rope, norm.q_w, norm.eps, stream);
  if (e == cudaSuccess && s == LC_OK)
    s = lc_rope_rows_bf16(k, k_rot, batch, N, heads, 0, rope, norm.k_w, norm.eps, stream);
  if (e == cudaSuccess && s == LC_OK)
    s = lc_bwd_delta(out, dout, delta, batch, N, heads, LC_DTYPE_BF16, stream);
  if (e == cudaSuccess && s == LC_OK) s = lc_encode_f32_halfrows(&prm.tmDQ, dq_acc, batch, N, heads);
  const void *src[4] = {q_rot, k_rot, v, dout};
  CUtensorMap *maps[4] = {prm.tmQ, prm.tmK, prm.tmV, prm.tmG};
  for (int i = 0; i < 4 && e == cudaSuccess && s == LC_OK; ++i) {
    s = lc_encode_segment(&maps[i][1], src[i], batch, N, Nc, Nn, heads);
    if (s == LC_OK && Nc > 0) s = lc_encode_segment(&maps[i][0], src[i], batch, N, 0, Nc, heads);
    if (Nc == 0) maps[i][0] = maps[i][1];  // unused, kept a valid descriptor
  }
  if (e == cudaSuccess && s == LC_OK) {
    prm.rope_tab = rope->tab;
    prm.kg_ptr = plan->kgrp_ptr;
    prm.kg_ent = plan->kgrp_ent;
    prm.kg_order = plan->kgrp_order;
    prm.kg_blk = plan->kgrp_blk;
    prm.lse = lse;
    prm.delta = delta;
    prm.dq_acc = dq_acc;
    prm.dk_acc = dk_acc;
    prm.work_counter = counter;
    prm.dk = static_cast<__nv_bfloat16 *>(dk);
    prm.dv = static_cast<__nv_bfloat16 *>(dv);
    prm.timeout_ns = 2000000000LL;
    prm.div_hw = lc_make_divmod(rope->H * rope->W);
    prm.div_w = lc_make_divmod(rope->W);
    prm.T = rope->T; prm.H = rope->H; prm.W = rope->W;
    prm.Nc = (int)Nc; prm.Nn = (int)Nn; prm.Cb = plan->Cb; prm.kgc = plan->kgc;
    prm.heads = heads;
    prm.KG = plan->KG;
    prm.n_blocks = plan->Cb + plan->Nb;
    prm.ent_cap = (int)plan->nnz;
    prm.total_items = (int)total;
    prm.tab_floats = tab_in_smem ? (int)rope->n_floats : 0;
    prm.scale = scale;
    const int grid = (int)(total < n_sm ? total : n_sm);
    kern<<<grid, kThreads, smem, stream>>>(prm);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess && s == LC_OK)
    s = lc_bwd_grad_finalize(dq_acc, q, dq, batch, N, heads, LC_DTYPE_BF16, norm.q_w, norm.eps,
                             rope, stream);
  if (e == cudaSuccess && s == LC_OK && dk_acc)
    s = lc_bwd_grad_finalize(dk_acc, k, dk, batch, N, heads, LC_DTYPE_BF16, norm.k_w, norm.eps,
                             rope, stream);
  if (dk_acc) cudaFreeAsync(dk_acc, stream);
  if (k_rot) cudaFreeAsync(k_rot, stream);
  if (q_rot) cudaFreeAsync(q_rot, stream);
  if (counter) cudaFreeAsync(counter, stream);
  if (dq_acc) cudaFreeAsync(dq_acc, stream);
  if (delta) cudaFreeAsync(delta, stream);
  if (s != LC_OK) return s;
  return lc_from_cuda(e);
}
