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
//   warp 8      TMA producer: Q tiles (double-buffered across items), then the
//               listed K and V blocks into a 3-stage ring (a missing second
//               block is an out-of-range box, which TMA fills with zeros).
//   warps 10-11 RoPE: rotate every freshly loaded Q tile, and K tile unless K
//               was rotated beforehand, in shared memory (128-byte swizzled
//               rows, cos/sin tables in smem), one token row per thread.
//   warp 9      MMA issuer (one thread): S_i = Q_i K^T (M=128, N=128, K=64)
//               into TMEM, O_i += P_i V (A = P from TMEM, M=128, N=64).
//   warps 0-3 / 4-7  softmax of Q0 / Q1, one TMEM lane (= query row) per
//               thread: mask, running max with lazy rescaling (threshold 2^8),
//               exp2 (part on the MUFU unit, part as a polynomial on the FMA
//               pipe), packed f32x2 sums, P as bf16 into TMEM; at the end
//               O / l through shared memory to a TMA store, plus the LSE.
//   TMEM (512 columns): three S buffers [0,128) [128,256) [256,384) taken
//               in turn by the (tile, warpgroup) sequence, each tile's P
//               written as bf16 over the first 64 columns of its own S
//               buffer; O0 [384,448) O1 [448,512).
// Launch modes (lc_fwd_mode): the whole sequence; the noisy queries with the
// condition K/V from separate tensors (cache consumer); the condition queries
// alone (cache producer); one shard pair of ring context parallelism (q / out
// and k / v hold token ranges of the sequence, addressed through per-segment
// tensor maps and row offsets; q and k may arrive rotated).
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
#include "sm100_sync.cuh"
#include "sm100_rope.cuh"
#include "sm100_math.cuh"

namespace {

#ifndef LC_KV_STAGES
#define LC_KV_STAGES 3
#endif
constexpr int kStages = LC_KV_STAGES;
// 1: a K/V ring stage has one "full" barrier (K and V bytes together) and one
// "empty" barrier (released after the stage's last P*V), which saves the MMA
// issuer a wait and a commit per tile; 0: separate K and V barriers.
#ifndef LC_KV_MERGED
#define LC_KV_MERGED 1
#endif
constexpr bool kKVMerged = LC_KV_MERGED != 0;
constexpr int kThreads = 384;
constexpr int kWarpProducer = 8;
constexpr int kWarpMma = 9;
constexpr int kWarpRope = 10;  // and 11
constexpr int kRopeThreads = 64;
constexpr int kTileBytes = 128 * 128;  // 128 rows x 64 bf16
constexpr int kBoxBytes = 64 * 128;    // one 64-row TMA box
constexpr uint32_t kTmemCols = 512;
// 1: three S buffers [0,128) [128,256) [256,384) taken in turn by the
// (tile, warpgroup) sequence, each tile's P written as bf16 over the first 64
// columns of its own S buffer, O0 [384,448) O1 [448,512): the next S never
// waits for a warpgroup to load its current one, and P never waits for the
// previous P*V (its buffer was last read by the P*V three positions back,
// which the tensor pipe executed before this tile's S).  0: two S buffers
// S0 [0,128) S1 [128,256), O0 [256,320) O1 [320,384), P0 [384,448) P1 [448,512).
#ifndef LC_S3
#define LC_S3 1
#endif
constexpr bool kS3 = LC_S3 != 0;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = kS3 ? 384 : 256, kColO1 = kS3 ? 448 : 320,
                   kColP0 = 384, kColP1 = 448;
constexpr uint32_t kIdescQK = lcptx::idesc_bf16_f32(128, 128, 0, 0);
constexpr uint32_t kIdescPV = lcptx::idesc_bf16_f32(128, 64, 0, 1);
constexpr float kRescaleThreshold = 8.0f;  // log2 units: p stays below 2^8 before a rescale
#ifndef LC_REGS_SOFTMAX
#define LC_REGS_SOFTMAX 200
#define LC_REGS_OTHER 104
#endif
constexpr int kRegsSoftmax = LC_REGS_SOFTMAX, kRegsOther = LC_REGS_OTHER;
static_assert(2 * 128 * LC_REGS_SOFTMAX + 128 * LC_REGS_OTHER <= 65536, "register split");
// Registers per thread the kernel must be launched with for that split.
constexpr int kRegsAtLaunchMin = (256 * kRegsSoftmax + 128 * kRegsOther + kThreads - 1) / kThreads;
// Of every 8 column pairs of a row, the pairs whose bit is set here take the
// polynomial exp2 on the FMA pipe; the others take MUFU ex2.
#ifndef LC_POLY_EXP2_MASK
#define LC_POLY_EXP2_MASK 0x00u
#endif
constexpr uint32_t kPolyMask = LC_POLY_EXP2_MASK;
// exp pass shape: pairs in flight between ex2 and their use (kLag <= kRing),
// and whether all logits are formed before the ex2 stream starts.
#ifndef LC_PASS_LAG
#define LC_PASS_LAG 2
#endif
#ifndef LC_LOGITS_FIRST
#define LC_LOGITS_FIRST 1
#endif
constexpr int kLag = LC_PASS_LAG, kRing = 16;
constexpr bool kLogitsFirst = LC_LOGITS_FIRST != 0;
static_assert(kLag <= kRing, "exp pass ring");

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
  int n_groups;            // groups of the plan (valid group ids: [0, n_groups))
  int n_blocks;            // key blocks of the pattern (valid key block ids: [0, n_blocks))
  int ent_cap;             // entries grp_ent holds (valid list bounds: [0, ent_cap])
  int group_offset;        // first rank of grp_order this launch works on
  int lse_nq;              // rows of the lse tensor per (batch, head)
  int lse_base[2];         // lse row of segment row 0, per segment ([0] condition, [1] noisy)
  int q_row_off[2];        // row of the q/out maps' row 0 within its segment (shards)
  int k_row_off[2];        // same for the k/v maps
  int tab_floats;
  int k_prerotated;        // K tensors already hold R(k): skip the K rotation
  int q_prerotated;        // Q tensors already hold R(q): skip the Q rotation (shards)
  float scale_log2;
  const float *q_norm_w;   // RMSNorm weights [64] applied ahead of the rotation, or NULL
  const float *k_norm_w;
  float norm_eps;
  // Programmatic dependent launch (shard steps of a ring): the next kernel on
  // the stream may launch once every CTA is set up, and this grid does not
  // finish before the previous one.  exit_counter (with work_counter, the
  // plan's own pair) counts finished CTAs; the last one resets both to 0.
  int pdl;
  int *exit_counter;
};

// Shared memory carve-up (offsets from a 1024-aligned base).
struct SmemOffsets {
  static constexpr int q = 0;                                  // [2 items][2 tiles]
  static constexpr int k = q + 4 * kTileBytes;                 // kStages tiles
  static constexpr int v = k + kStages * kTileBytes;           // kStages tiles
  static constexpr int bars = v + kStages * kTileBytes;        // mbarriers
  static constexpr int n_bars = 64;
  static constexpr int misc = bars + n_bars * 8;               // tmem base, items, abort
  static constexpr int normw = misc + 64;                      // q, k RMSNorm weights (fp32)
  static constexpr int tab = normw + 2 * 64 * 4;               // rope tables (fp32)
};

// Barrier indices.
enum {
  B_QFULL = 0,    // [buf*2 + i] TMA Q landed
  B_QREADY = 4,   // [buf*2 + i] Q rotated
  B_QEMPTY = 8,   // [buf*2 + i] Q buffer (and O staging) free
  B_KFULL = 12,   // [kStages]
  B_KREADY = B_KFULL + kStages,
  B_KEMPTY = B_KFULL + 2 * kStages,
  B_VFULL = B_KFULL + 3 * kStages,
  B_VEMPTY = B_KFULL + 4 * kStages,
  B_SFULL = B_KFULL + 5 * kStages,  // [2] per warpgroup, or [3] per S buffer (kS3)
  B_SFREE = B_SFULL + 3,            // [2] (not with kS3)
  B_PFULL = B_SFREE + 2,            // [2]
  B_ODONE = B_PFULL + 2,            // [2]
  B_EPI = B_ODONE + 2,              // [2] O rows staged in smem
  B_SCHED_FULL = B_EPI + 2,         // [2]
  B_SCHED_EMPTY = B_SCHED_FULL + 2, // [2]
  B_DRAIN = B_SCHED_EMPTY + 2,
  B_COUNT = B_DRAIN + 1
};
static_assert(B_COUNT <= SmemOffsets::n_bars, "barrier space");
constexpr int kSchedConsumers = 8 + 1 + 2;  // softmax warps, MMA warp, RoPE warps

using lcsm100::Ctx;
using lcsm100::wait_bar;
using lcsm100::wait_warp;

struct Item {
  int b, h, seg, row0, seg_len, len;
  const uint32_t *ent;
};

// Device-side plan checks: a group id, list bound or entry that a consistent
// plan never holds is replaced by a harmless one (group 0, a one-entry list,
// an absent key block that loads as zeros and is fully masked) before it is
// used as an index or a TMA coordinate, and LC_DEVSTAT_CHECK is raised by the
// role passed `status` (the producer), so that every role of the CTA takes
// the same decision and the host learns of it from lc_last_device_status.
__device__ __forceinline__ Item decode_item(const Sm100Params &p, int item, int *status) {
  Item it;
  int per = p.n_groups_active;
  int bh = item / per;
  int g = p.grp_order[p.group_offset + item - bh * per];
  bool bad = (unsigned)g >= (unsigned)p.n_groups;
  if (bad) g = 0;
  it.b = bh / p.heads;
  it.h = bh - it.b * p.heads;
  it.seg = g < p.gc ? 0 : 1;
  int qb0 = it.seg ? 4 * (g - p.gc) : 4 * g;
  it.row0 = 64 * qb0;
  it.seg_len = it.seg ? p.Nn : p.Nc;
  int lo = p.grp_ptr[g], hi = p.grp_ptr[g + 1];
  if (lo < 0 || hi <= lo || hi > p.ent_cap) {
    bad = true;
    lo = 0;
    hi = 1;
  }
  it.len = hi - lo;
  it.ent = p.grp_ent + lo;
  if (bad && status) atomicOr(status, LC_DEVSTAT_CHECK);
  return it;
}

// A plan entry names a key block of the pattern and at least one member.
__device__ __forceinline__ bool entry_ok(const Sm100Params &p, uint32_t e) {
  return (int)(e & 0xFFFFFFu) < p.n_blocks && ((e >> 24) - 1u) < 15u;
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

// Entries of an item's list, fetched 32 at a time by a whole warp: lane i
// holds entry 32*chunk + i; the next chunk is prefetched one chunk ahead.
struct EntryStream {
  uint32_t cur, nxt;
  int len;
  const uint32_t *ent;
  __device__ __forceinline__ void start(const uint32_t *e, int n, int lane) {
    ent = e;
    len = n;
    cur = lane < n ? __ldg(e + lane) : 0u;
    nxt = 32 + lane < n ? __ldg(e + 32 + lane) : 0u;
  }
  // Entries 2t and 2t+1 (the second is 0 past the end).
  __device__ __forceinline__ void pair(int t, int lane, uint32_t &a, uint32_t &b) {
    const int i = (2 * t) & 31;
    if (t > 0 && i == 0) {
      cur = nxt;
      const int j = 2 * t + 32 + lane;
      nxt = j < len ? __ldg(ent + j) : 0u;
    }
    a = __shfl_sync(0xffffffffu, cur, i);
    b = __shfl_sync(0xffffffffu, cur, i + 1);
    if (2 * t + 1 >= len) b = 0u;
  }
};

__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

using lcsm100::rope_row;
using lcsm100::rot_chunk_bf16;
using lcsm100::sumsq_chunk_bf16;

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

// Maximum of a 128-column score row: 8 independent chains of 3-input maxima.
__device__ __forceinline__ float row_max(const float (&s)[128]) {
  float mc[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) mc[c] = fmaxf(s[2 * c], s[2 * c + 1]);
#pragma unroll
  for (int j = 16; j < 128; j += 16)
#pragma unroll
    for (int c = 0; c < 8; ++c) mc[c] = max3(mc[c], s[j + 2 * c], s[j + 2 * c + 1]);
  return max3(max3(mc[0], mc[1], mc[2]), max3(mc[3], mc[4], mc[5]), fmaxf(mc[6], mc[7]));
}

// Mask limits of tile tt of an item for the rows of query block `qsub`:
// bits 0-7 = attended tokens of the tile's first key block (0 when the block
// is not attended), bits 8-15 = same for the second block.
__device__ __forceinline__ uint32_t tile_limits(const Sm100Params &p, const Item &it, int tt,
                                                int qsub) {
  // (an entry that fails the plan check only gives a mask here; the
  // producer reports it and loads zeros for it)
  if (2 * tt >= it.len) return 0u;
  const uint32_t ea = __ldg(it.ent + 2 * tt);
  int sx, rx, na, nb = 0;
  entry_block(p, ea, sx, rx, na);
  if (!((ea >> (24 + qsub)) & 1u)) na = 0;
  if (2 * tt + 1 < it.len) {
    const uint32_t eb = __ldg(it.ent + 2 * tt + 1);
    entry_block(p, eb, sx, rx, nb);
    if (!((eb >> (24 + qsub)) & 1u)) nb = 0;
  }
  return (uint32_t)na | ((uint32_t)nb << 8);
}

// kQKNorm: the RoPE warps apply the RMSNorm weights of p (instantiated
// separately so that the plain path carries no trace of it).
template <bool kQKNorm>
__global__ void __launch_bounds__(kThreads, 1) bsa_sm100_kernel(const __grid_constant__ Sm100Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  uint8_t *sQ = smem + SmemOffsets::q;  // tile (buf, i) at sQ + (2*buf + i) * kTileBytes
  uint8_t *sK = smem + SmemOffsets::k;
  uint8_t *sV = smem + SmemOffsets::v;
  uint32_t *misc = reinterpret_cast<uint32_t *>(smem + SmemOffsets::misc);
  // misc[0] tmem base, misc[1..2] scheduled items, misc[3] abort flag
  float *tab = reinterpret_cast<float *>(smem + SmemOffsets::tab);
  float *s_normw = reinterpret_cast<float *>(smem + SmemOffsets::normw);  // [q 64 | k 64]
  Ctx ctx;
  ctx.bar0 = lcptx::smem_addr(smem + SmemOffsets::bars);
  ctx.abort_flag = reinterpret_cast<volatile int *>(&misc[3]);
  ctx.status = p.status;
  ctx.timeout_ns = p.timeout_ns;

  // ---- set-up: tables, barriers, TMEM
  for (int i = tid; i < p.tab_floats; i += kThreads) tab[i] = p.rope_tab[i];
  if (tid < 64 && p.q_norm_w) s_normw[tid] = p.q_norm_w[tid];
  if (tid < 64 && p.k_norm_w) s_normw[64 + tid] = p.k_norm_w[tid];
  if (tid == 0) {
    misc[3] = 0;
    for (int i = 0; i < 4; ++i) {
      lcptx::mbar_init(ctx.bar(B_QFULL + i), 1);
      lcptx::mbar_init(ctx.bar(B_QREADY + i), kRopeThreads);
      lcptx::mbar_init(ctx.bar(B_QEMPTY + i), 1);
    }
    lcptx::mbar_init(ctx.bar(B_SFULL + 2), 1);
    for (int i = 0; i < 2; ++i) {
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
  const bool k_rot = p.k_prerotated != 0;
  if (p.pdl) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // Register split: the softmax warpgroups (warps 0-7) hold a 128-column row
  // of S in registers; the producer / MMA / RoPE warpgroup needs few.
  // 256 x kRegsSoftmax + 128 x kRegsOther must not exceed the registers the
  // block was launched with; the host refuses to launch otherwise.
  if (warp >= 8) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsOther));
  if (warp == kWarpProducer) {
    // ======================= TMA producer (one thread) =======================
    if (lane == 0) {
      uint32_t kv_it = 0, item_it = 0;
      // Issued loads, for the drain: bit j of *_valid says barrier j got a
      // load, bit j of *_par is the parity of its last phase.
      uint32_t q_valid = 0, q_par = 0, k_valid = 0, k_par = 0, v_valid = 0, v_par = 0;
      for (;;) {
        const int slot = item_it & 1;
        int item = atomicAdd(p.work_counter, 1);
        if (item >= p.total_items) item = -1;
        if (!wait_bar(ctx, ctx.bar(B_SCHED_EMPTY + slot), ((item_it >> 1) & 1) ^ 1)) break;
        misc[1 + slot] = (uint32_t)item;
        lcptx::mbar_arrive(ctx.bar(B_SCHED_FULL + slot));
        if (item < 0) break;
        const Item it = decode_item(p, item, p.status);
        const int buf = item_it & 1;
        const uint32_t qph = (item_it >> 1) & 1;
        bool ok = true;
        for (int i = 0; i < 2 && ok; ++i) {
          const int qi = 2 * buf + i;
          ok = wait_bar(ctx, ctx.bar(B_QEMPTY + qi), qph ^ 1);
          if (!ok) break;
          const uint32_t bq = ctx.bar(B_QFULL + qi);
          lcptx::mbar_arrive_expect_tx(bq, kTileBytes);
          const uint32_t dst = lcptx::smem_addr(sQ + qi * kTileBytes);
          const int r = it.row0 + 128 * i - p.q_row_off[it.seg];
          lcptx::tma_load_4d(dst, &p.tmQ[it.seg], bq, 0, it.h, r, it.b);
          lcptx::tma_load_4d(dst + kBoxBytes, &p.tmQ[it.seg], bq, 0, it.h, r + 64, it.b);
          q_valid |= 1u << qi;
          q_par = (q_par & ~(1u << qi)) | (qph << qi);
        }
        if (!ok) break;
        const int ntiles = (it.len + 1) >> 1;
        for (int t = 0; t < ntiles && ok; ++t, ++kv_it) {
          const int s = kv_it % kStages;
          const uint32_t ph = (kv_it / kStages) & 1;
          // a missing second block, or an entry that fails the plan check, is a
          // box far past every map's end: it reads zeros (and is masked)
          int sa = 1, ra = 1 << 24, na, sb = 1, rb = 1 << 24, nb;
          const uint32_t ea = __ldg(it.ent + 2 * t);
          if (entry_ok(p, ea)) {
            entry_block(p, ea, sa, ra, na);
            ra -= p.k_row_off[sa];
          } else {
            atomicOr(p.status, LC_DEVSTAT_CHECK);
          }
          if (2 * t + 1 < it.len) {
            const uint32_t eb = __ldg(it.ent + 2 * t + 1);
            if (entry_ok(p, eb)) {
              entry_block(p, eb, sb, rb, nb);
              rb -= p.k_row_off[sb];
            } else {
              atomicOr(p.status, LC_DEVSTAT_CHECK);
            }
          }
          ok = wait_bar(ctx, ctx.bar(B_KEMPTY + s), ph ^ 1);
          if (!ok) break;
          const uint32_t bk = ctx.bar(B_KFULL + s);
          lcptx::mbar_arrive_expect_tx(bk, kKVMerged ? 2 * kTileBytes : kTileBytes);
          const uint32_t dk = lcptx::smem_addr(sK + s * kTileBytes);
          lcptx::tma_load_4d(dk, &p.tmK[sa], bk, 0, it.h, ra, it.b);
          lcptx::tma_load_4d(dk + kBoxBytes, &p.tmK[sb], bk, 0, it.h, rb, it.b);
          k_valid |= 1u << s;
          k_par = (k_par & ~(1u << s)) | (ph << s);
          if (!kKVMerged) ok = wait_bar(ctx, ctx.bar(B_VEMPTY + s), ph ^ 1);
          if (!ok) break;
          const uint32_t bv = ctx.bar(kKVMerged ? B_KFULL + s : B_VFULL + s);
          if (!kKVMerged) lcptx::mbar_arrive_expect_tx(bv, kTileBytes);
          const uint32_t dv = lcptx::smem_addr(sV + s * kTileBytes);
          lcptx::tma_load_4d(dv, &p.tmV[sa], bv, 0, it.h, ra, it.b);
          lcptx::tma_load_4d(dv + kBoxBytes, &p.tmV[sb], bv, 0, it.h, rb, it.b);
          if (!kKVMerged) {
            v_valid |= 1u << s;
            v_par = (v_par & ~(1u << s)) | (ph << s);
          }
        }
        if (!ok) break;
        ++item_it;
      }
      // Drain: every load this thread issued must land before the CTA exits.
      auto drain = [&](uint32_t bar, uint32_t valid, uint32_t par, int j) {
        if (!((valid >> j) & 1u)) return;
        const uint32_t ph = (par >> j) & 1u;
        const uint64_t t0 = lcptx::globaltimer_ns();
        while (!lcptx::mbar_try_wait(bar, ph) &&
               (long long)(lcptx::globaltimer_ns() - t0) < p.timeout_ns) {
        }
      };
#pragma unroll
      for (int i = 0; i < 4; ++i) drain(ctx.bar(B_QFULL + i), q_valid, q_par, i);
#pragma unroll
      for (int s = 0; s < kStages; ++s) {
        drain(ctx.bar(B_KFULL + s), k_valid, k_par, s);
        drain(ctx.bar(B_VFULL + s), v_valid, v_par, s);
      }
    }
  } else if (warp == kWarpMma) {
    // ======================= MMA issuer (one thread) =========================
    if (lane == 0) {
      uint32_t item_it = 0;
      int cs = 0;        // K/V stage of the current tile
      uint32_t cph = 0;  // and its phase parity
      uint32_t sfree_bits = 0, pfull_bits = 0;  // bit i: phase parity for tile i
      uint32_t kpos = 0;  // (tile, warpgroup) position of the item's tile 0, warpgroup 0
      const int kbar = k_rot ? B_KFULL : B_KREADY;
      // Operand descriptors, built once: the high word (stride byte offset
      // 1024, version 1, 128-byte swizzle) is common; the low word holds the
      // start address >> 4 and the leading byte offset, and steps by 32 bytes
      // per 16-wide K slice of Q/K and by 2048 bytes (16 keys) for V.
      constexpr uint32_t kDescHi = (1024u >> 4) | (1u << 14) | (2u << 29);
      constexpr uint32_t kTileLo = kTileBytes >> 4;
      const uint32_t q_lo0 = (lcptx::smem_addr(sQ) >> 4) | (1u << 16);
      const uint32_t k_lo0 = (lcptx::smem_addr(sK) >> 4) | (1u << 16);
      const uint32_t v_lo0 = (lcptx::smem_addr(sV) >> 4) | (512u << 16);
      auto desc = [](uint32_t lo) -> uint64_t {
        return (static_cast<uint64_t>(kDescHi) << 32) | lo;
      };
      for (;;) {
        const int slot = item_it & 1;
        if (!wait_bar(ctx, ctx.bar(B_SCHED_FULL + slot), (item_it >> 1) & 1)) break;
        const int item = (int)misc[1 + slot];
        lcptx::mbar_arrive(ctx.bar(B_SCHED_EMPTY + slot));
        if (item < 0) break;
        const Item it = decode_item(p, item, nullptr);
        const int ntiles = (it.len + 1) >> 1;
        const int buf = item_it & 1;
        const uint32_t qph = (item_it >> 1) & 1;
        bool ok = wait_bar(ctx, ctx.bar(B_QREADY + 2 * buf), qph) &&
                  wait_bar(ctx, ctx.bar(B_QREADY + 2 * buf + 1), qph);
        if (!ok) break;
        const uint32_t q_lo = q_lo0 + 2 * buf * kTileLo;
        // k: the (tile, warpgroup) position; with kS3 its S buffer is k % 3.
        auto issue_s = [&](int i, int s, uint32_t k) -> bool {
          uint32_t d, bar;
          if (kS3) {
            d = tmem + 128u * (k % 3u);
            bar = ctx.bar(B_SFULL + (int)(k % 3u));
          } else {
            if (!wait_bar(ctx, ctx.bar(B_SFREE + i), ((sfree_bits >> i) & 1u) ^ 1u)) return false;
            sfree_bits ^= 1u << i;
            d = tmem + (i ? kColS1 : kColS0);
            bar = ctx.bar(B_SFULL + i);
          }
          lcptx::tc_fence_after();
          const uint32_t qa = q_lo + i * kTileLo, kb = k_lo0 + s * kTileLo;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            lcptx::mma_ss(d, desc(qa + 2 * kk), desc(kb + 2 * kk), kIdescQK, kk > 0);
          lcptx::mma_commit(bar);
          return true;
        };
        auto issue_pv = [&](int i, int s, bool accumulate, uint32_t k) -> bool {
          if (!wait_bar(ctx, ctx.bar(B_PFULL + i), (pfull_bits >> i) & 1u)) return false;
          pfull_bits ^= 1u << i;
          lcptx::tc_fence_after();
          const uint32_t vb = v_lo0 + s * kTileLo;
          const uint32_t d = tmem + (i ? kColO1 : kColO0);
          const uint32_t a = kS3 ? tmem + 128u * (k % 3u) : tmem + (i ? kColP1 : kColP0);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            lcptx::mma_ts(d, a + 8 * kk, desc(vb + 128 * kk), kIdescPV,
                          (accumulate || kk > 0) ? 1u : 0u);
          lcptx::mma_commit(ctx.bar(B_ODONE + i));
          return true;
        };
        // tile 0: both S tiles
        const uint32_t k0 = kpos;
        ok = wait_bar(ctx, ctx.bar(kbar + cs), cph) && issue_s(0, cs, k0) && issue_s(1, cs, k0 + 1);
        if (!ok) break;
        if (!kKVMerged) lcptx::mma_commit(ctx.bar(B_KEMPTY + cs));
        for (int t = 0; t < ntiles && ok; ++t) {
          const bool more = t + 1 < ntiles;
          const int ns = cs + 1 == kStages ? 0 : cs + 1;
          const uint32_t nph = ns == 0 ? cph ^ 1u : cph;
          const uint32_t kt = k0 + 2u * (uint32_t)t;
          if (more) {
            ok = wait_bar(ctx, ctx.bar(kbar + ns), nph) && issue_s(0, ns, kt + 2);
            if (!ok) break;
          }
          ok = (kKVMerged || wait_bar(ctx, ctx.bar(B_VFULL + cs), cph)) &&
               issue_pv(0, cs, t > 0, kt);
          if (!ok) break;
          if (more) {
            ok = issue_s(1, ns, kt + 3);
            if (!ok) break;
            if (!kKVMerged) lcptx::mma_commit(ctx.bar(B_KEMPTY + ns));
          }
          ok = issue_pv(1, cs, t > 0, kt + 1);
          if (!ok) break;
          lcptx::mma_commit(ctx.bar(kKVMerged ? B_KEMPTY + cs : B_VEMPTY + cs));
          cs = ns;
          cph = nph;
        }
        if (!ok) break;
        kpos = k0 + 2u * (uint32_t)ntiles;
        ++item_it;
      }
      // Drain: wait until every MMA this thread issued has completed.
      lcptx::mma_commit(ctx.bar(B_DRAIN));
      const uint64_t t0 = lcptx::globaltimer_ns();
      while (!lcptx::mbar_try_wait(ctx.bar(B_DRAIN), 0) &&
             (long long)(lcptx::globaltimer_ns() - t0) < p.timeout_ns) {
      }
    }
    __syncwarp();
  } else {
    // ======================= RoPE warps ======================================
    const int rt = tid - kWarpRope * 32;
    const float *q_nw = (kQKNorm && p.q_norm_w) ? s_normw : nullptr;
    const float *k_nw = (kQKNorm && p.k_norm_w) ? s_normw + 64 : nullptr;
    uint32_t item_it = 0, kv_it = 0;
    EntryStream es;
    for (;;) {
      const int slot = item_it & 1;
      if (!wait_warp(ctx, ctx.bar(B_SCHED_FULL + slot), (item_it >> 1) & 1)) break;
      const int item = (int)misc[1 + slot];
      __syncwarp();
      if (lane == 0) lcptx::mbar_arrive(ctx.bar(B_SCHED_EMPTY + slot));
      if (item < 0) break;
      const Item it = decode_item(p, item, nullptr);
      const int seg_base = it.seg ? p.Nc : 0;  // sequence index of the segment's token 0
      const int buf = item_it & 1;
      const uint32_t qph = (item_it >> 1) & 1;
      bool ok = true;
      for (int i = 0; i < 2 && ok; ++i) {
        const int qi = 2 * buf + i;
        ok = wait_warp(ctx, ctx.bar(B_QFULL + qi), qph);
        if (!ok) break;
        const int r0 = it.row0 + 128 * i;
        const int nrows = p.q_prerotated ? 0 : min(128, it.seg_len - r0);
#pragma unroll 1
        for (int r = rt; r < nrows; r += kRopeThreads)
          rope_row(sQ + qi * kTileBytes, r, seg_base + r0 + r, tab, p, q_nw);
        lcptx::fence_proxy_async_smem();
        lcptx::mbar_arrive(ctx.bar(B_QREADY + qi));
      }
      if (!ok) break;
      if (!k_rot) {
        const int ntiles = (it.len + 1) >> 1;
        es.start(it.ent, it.len, lane);
        for (int t = 0; t < ntiles; ++t, ++kv_it) {
          const int s = kv_it % kStages;
          uint32_t ea, eb;
          es.pair(t, lane, ea, eb);
          ok = wait_warp(ctx, ctx.bar(B_KFULL + s), (kv_it / kStages) & 1);
          if (!ok) break;
          uint8_t *tile = sK + s * kTileBytes;
          // Row rt of each of the tile's two key blocks (one code copy).
#pragma unroll 1
          for (int half = 0; half < 2; ++half) {
            if (half == 1 && 2 * t + 1 >= it.len) break;
            const uint32_t ex = half ? eb : ea;
            if (!entry_ok(p, ex)) continue;
            int sx, rx, nx;
            entry_block(p, ex, sx, rx, nx);
            if (rt < nx) rope_row(tile, 64 * half + rt, (sx ? p.Nc : 0) + rx + rt, tab, p, k_nw);
          }
          lcptx::fence_proxy_async_smem();
          lcptx::mbar_arrive(ctx.bar(B_KREADY + s));
        }
        if (!ok) break;
      }
      ++item_it;
    }
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    // ======================= softmax warpgroups ==============================
    const int wg = warp >> 2;              // which Q tile
    const int row = tid & 127;             // TMEM lane == tile row
    const int qsub = 2 * wg + (row >> 6);  // member index of this row's query block
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tO = tmem + lane_base + (wg ? kColO1 : kColO0);
    const float sl2 = p.scale_log2;
    uint32_t item_it = 0, sfull_ph = 0, odone_ph = 0;
    // kS3: this warpgroup's next (tile, warpgroup) position and the P*V
    // products issued for it so far (ODONE completes once per product; a
    // wait for the latest one takes its parity from this count).
    uint32_t kpos = (uint32_t)wg, n_pv = 0;
    for (;;) {
      const int slot = item_it & 1;
      if (!wait_warp(ctx, ctx.bar(B_SCHED_FULL + slot), (item_it >> 1) & 1)) break;
      const int item = (int)misc[1 + slot];
      __syncwarp();
      if (lane == 0) lcptx::mbar_arrive(ctx.bar(B_SCHED_EMPTY + slot));
      if (item < 0) break;
      const Item it = decode_item(p, item, nullptr);
      const int ntiles = (it.len + 1) >> 1;
      // Mask limits of this warp's rows, one tile per lane, 32 tiles at a time.
      uint32_t lim_lane = 0;
      float m_ref = -INFINITY, l_sum = 0.f;
      bool ok = true;
      for (int t = 0; t < ntiles; ++t) {
        if ((t & 31) == 0) lim_lane = tile_limits(p, it, t + lane, qsub);
        const uint32_t lim = __shfl_sync(0xffffffffu, lim_lane, t & 31);
        const int na = lim & 0xFF, nb = (lim >> 8) & 0xFF;
        // This tile's S (and, with kS3, its P) columns.
        const uint32_t buf = kS3 ? kpos % 3u : 0u;
        const uint32_t tS = tmem + lane_base + (kS3 ? 128u * buf : (wg ? kColS1 : kColS0));
        const uint32_t tP = kS3 ? tS : tmem + lane_base + (wg ? kColP1 : kColP0);
        if (kS3) {
          ok = wait_warp(ctx, ctx.bar(B_SFULL + (int)buf), (kpos / 3u) & 1u);
        } else {
          ok = wait_warp(ctx, ctx.bar(B_SFULL + wg), sfull_ph);
          sfull_ph ^= 1;
        }
        if (!ok) break;
        lcptx::tc_fence_after();
        uint32_t r0[32], r1[32], r2[32], r3[32];
        lcptx::tmem_ld32(tS, r0);
        lcptx::tmem_ld32(tS + 32, r1);
        lcptx::tmem_ld32(tS + 64, r2);
        lcptx::tmem_ld32(tS + 96, r3);
        lcptx::tmem_wait_ld();
        lcptx::tc_fence_before();
        __syncwarp();
        if (!kS3 && lane == 0) lcptx::mbar_arrive(ctx.bar(B_SFREE + wg));
        float s[128];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          s[j] = __uint_as_float(r0[j]);
          s[32 + j] = __uint_as_float(r1[j]);
          s[64 + j] = __uint_as_float(r2[j]);
          s[96 + j] = __uint_as_float(r3[j]);
        }
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
        // The first tile sets the reference max exactly.  Later tiles reuse
        // it: P = 2^(x) with x = s * scale_log2 - m_ref and no row max at all,
        // which is valid as long as no element exceeds m_ref + 8 -- certain
        // when the tile's sum is at most 2^8.  Otherwise the row max is taken,
        // and if it is above m_ref + 8 the reference moves up, O and l are
        // rescaled and P is redone from the logits kept in s.
        if (t == 0) m_ref = row_max(s) * sl2;
        float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
        // P / O of this warpgroup free (previous P*V done); with kS3 P goes
        // to a buffer no product reads any more, so only O needs the wait.
        bool o_ready = kS3 || t == 0;
        float l_tile = 0.f;
        // One pass: s <- s * mul + add in place, P = 2^s pipelined (the ex2 of
        // pair j is issued after pair j-8 is packed and summed), P to TMEM in
        // 32-key chunks; waits for the previous P*V just before the first store.
        auto pass = [&](float mul, float add) -> bool {
          const float2 mul2 = make_float2(mul, mul), add2 = make_float2(add, add);
          float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                           make_float2(0.f, 0.f)};
          float e[2 * kRing];
          uint32_t pk[16];
          if (kLogitsFirst) {  // all 64 FFMA2 up front, independent of the ex2 stream
#pragma unroll
            for (int j = 0; j < 64; ++j) {
              const float2 x = __ffma2_rn(make_float2(s[2 * j], s[2 * j + 1]), mul2, add2);
              s[2 * j] = x.x;
              s[2 * j + 1] = x.y;
            }
          }
#pragma unroll
          for (int j = 0; j < 64 + kLag; ++j) {
            if (j >= kLag) {  // consume pair k = j - kLag
              const int k = j - kLag;
              const float2 v = make_float2(e[2 * (k & (kRing - 1))], e[2 * (k & (kRing - 1)) + 1]);
              acc[k & 3] = __fadd2_rn(acc[k & 3], v);
              pk[k & 15] = pack_bf16(v.x, v.y);
              if ((k & 15) == 15) {
                if (!o_ready) {
                  if (!wait_warp(ctx, ctx.bar(B_ODONE + wg), odone_ph)) return false;
                  odone_ph ^= 1;
                  lcptx::tc_fence_after();
                  o_ready = true;
                }
                lcptx::tmem_st16(tP + 16 * (k >> 4), pk);
              }
            }
            if (j < 64) {  // logits and ex2 of pair j
              float2 x = make_float2(s[2 * j], s[2 * j + 1]);
              if (!kLogitsFirst) {
                x = __ffma2_rn(x, mul2, add2);
                s[2 * j] = x.x;
                s[2 * j + 1] = x.y;
              }
              if (kPolyMask & (1u << (j & 7))) {
                const float2 y = lcsm100::exp2_poly2(x);
                e[2 * (j & (kRing - 1))] = y.x;
                e[2 * (j & (kRing - 1)) + 1] = y.y;
              } else {
                e[2 * (j & (kRing - 1))] = ex2(x.x);
                e[2 * (j & (kRing - 1)) + 1] = ex2(x.y);
              }
            }
          }
          const float2 a = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
          l_tile = a.x + a.y;
          return true;
        };
        ok = pass(sl2, -m_use);
        if (!ok) break;
        float alpha = 1.f;
        bool rescale_o = false;
        if (t > 0 && __any_sync(0xffffffffu, !(l_tile <= 256.f))) {
          const float mt = row_max(s) + m_use;  // s now holds logits minus m_use
          if (__any_sync(0xffffffffu, mt > m_ref + kRescaleThreshold)) {
            const float m_new = fmaxf(m_ref, mt);
            const float m_new_use = (m_new == -INFINITY) ? 0.f : m_new;
            // O and l so far are relative to m_use, which is 0 while the row
            // has met no attended key in an earlier tile (m_ref = -inf) -- a
            // group's first tile can be fully masked for some member rows.
            alpha = ex2(m_use - m_new_use);
            l_sum *= alpha;
            m_ref = m_new;
            ok = pass(1.f, m_use - m_new_use);
            if (!ok) break;
            m_use = m_new_use;
            rescale_o = true;
          }
        }
        if (!o_ready) {  // (a tile always stores P, so this is only a safeguard)
          ok = wait_warp(ctx, ctx.bar(B_ODONE + wg), odone_ph);
          if (!ok) break;
          odone_ph ^= 1;
          lcptx::tc_fence_after();
        }
        l_sum += l_tile;
        // kS3: the previous tile's P*V (issued about a pass ago) is waited for
        // before this tile's P is handed over, so that at most one product is
        // ever outstanding and a parity wait on ODONE is never two phases
        // behind; O may then be rescaled.
        if (kS3 && n_pv > 0) {
          ok = wait_warp(ctx, ctx.bar(B_ODONE + wg), (n_pv - 1u) & 1u);
          if (!ok) break;
          lcptx::tc_fence_after();
        }
        if (rescale_o) {
          uint32_t o0[32], o1[32];
          lcptx::tmem_ld32(tO, o0);
          lcptx::tmem_ld32(tO + 32, o1);
          lcptx::tmem_wait_ld();
          const float2 al = make_float2(alpha, alpha);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            float2 u = __fmul2_rn(make_float2(__uint_as_float(o0[2 * j]), __uint_as_float(o0[2 * j + 1])), al);
            float2 v = __fmul2_rn(make_float2(__uint_as_float(o1[2 * j]), __uint_as_float(o1[2 * j + 1])), al);
            o0[2 * j] = __float_as_uint(u.x); o0[2 * j + 1] = __float_as_uint(u.y);
            o1[2 * j] = __float_as_uint(v.x); o1[2 * j + 1] = __float_as_uint(v.y);
          }
          lcptx::tmem_st32(tO, o0);
          lcptx::tmem_st32(tO + 32, o1);
        }
        lcptx::tmem_wait_st();
        lcptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) lcptx::mbar_arrive(ctx.bar(B_PFULL + wg));
        ++n_pv;
        kpos += 2;
      }
      if (!ok) break;
      // ---- epilogue: O / l -> bf16 -> smem (swizzled) -> TMA store; lse
      if (kS3) {
        ok = wait_warp(ctx, ctx.bar(B_ODONE + wg), (n_pv - 1u) & 1u);
      } else {
        ok = wait_warp(ctx, ctx.bar(B_ODONE + wg), odone_ph);
        odone_ph ^= 1;
      }
      if (!ok) break;
      lcptx::tc_fence_after();
      const float inv_l = l_sum > 0.f ? 1.f / l_sum : 0.f;
      const int buf = item_it & 1;
      uint8_t *stage = sQ + (2 * buf + wg) * kTileBytes;
      {
        uint32_t o0[32], o1[32];
        lcptx::tmem_ld32(tO, o0);
        lcptx::tmem_ld32(tO + 32, o1);
        lcptx::tmem_wait_ld();
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint32_t *o = ch < 4 ? o0 + 8 * ch : o1 + 8 * (ch - 4);
          uint4 v;
          v.x = pack_bf16(__uint_as_float(o[0]) * inv_l, __uint_as_float(o[1]) * inv_l);
          v.y = pack_bf16(__uint_as_float(o[2]) * inv_l, __uint_as_float(o[3]) * inv_l);
          v.z = pack_bf16(__uint_as_float(o[4]) * inv_l, __uint_as_float(o[5]) * inv_l);
          v.w = pack_bf16(__uint_as_float(o[6]) * inv_l, __uint_as_float(o[7]) * inv_l);
          *reinterpret_cast<uint4 *>(stage + swz(row, ch)) = v;
        }
      }
      lcptx::tc_fence_before();
      const int qrow = it.row0 + 128 * wg + row;  // row within the segment
      if (p.lse && qrow < it.seg_len) {
        const int out_row = p.lse_base[it.seg] + qrow;
        p.lse[((long long)it.b * p.heads + it.h) * p.lse_nq + out_row] =
            ((m_ref == -INFINITY ? 0.f : m_ref) + __log2f(l_sum)) * 0.69314718055994530942f;
      }
      lcptx::fence_proxy_async_smem();
      lcptx::mbar_arrive(ctx.bar(B_EPI + wg));
      if (row == 0) {
        ok = wait_bar(ctx, ctx.bar(B_EPI + wg), item_it & 1);
        if (ok) {
          const uint32_t src = lcptx::smem_addr(stage);
          const int r0 = it.row0 + 128 * wg;  // row within the segment
          const int c0 = r0 - p.q_row_off[it.seg];  // row of the out map (>= 0: groups lie in the shard)
          if (r0 < it.seg_len) lcptx::tma_store_4d(&p.tmO[it.seg], src, 0, it.h, c0, it.b);
          if (r0 + 64 < it.seg_len)
            lcptx::tma_store_4d(&p.tmO[it.seg], src + kBoxBytes, 0, it.h, c0 + 64, it.b);
          lcptx::bulk_commit_group();
          lcptx::bulk_wait_group_read0();
          lcptx::mbar_arrive(ctx.bar(B_QEMPTY + 2 * buf + wg));
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
  if (tid == 0) {
    // Every producer has taken its last item: the last CTA out resets the
    // plan's scheduler for the next launch that uses it.
    if (p.exit_counter && atomicAdd(p.exit_counter, 1) == (int)gridDim.x - 1) {
      *p.work_counter = 0;
      *p.exit_counter = 0;
      __threadfence();
    }
    // Finish no earlier than the previous grid on the stream.
    if (p.pdl) asm volatile("griddepcontrol.wait;" ::: "memory");
  }
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

// Standalone rotation of K (or any [B, ntok, heads, 64] bf16 tensor) into a
// separate buffer, 16 bytes per thread step; used when the attention kernel
// is given K already rotated.  Same arithmetic as rope_row: with nw, the
// eight lanes that hold a row's chunks combine their sums of squares.
__global__ void rope_k_kernel(const uint4 *src, uint4 *dst, long long n_chunks, int heads,
                              long long ntok, int tok_offset, const float *tab, int T, int H,
                              int W, lc_divmod div_hw, lc_divmod div_w, const float *nw,
                              float eps) {
  const unsigned group = 0xFFu << (threadIdx.x & 24);  // this lane's 8-lane group
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n_chunks;
       i += (long long)gridDim.x * blockDim.x) {
    const int ch = (int)(i & 7);
    const long long tokhead = i >> 3;
    const int n = (int)((tokhead / heads) % ntok) + tok_offset;
    const int t = lc_div(n, div_hw);
    const int rem = n - t * div_hw.d;
    const int hh = lc_div(rem, div_w);
    const int w = rem - hh * div_w.d;
    const float *c, *s;
    if (ch < 2) { c = tab + t * 8 + 4 * ch; s = c + T * 8; }
    else if (ch < 5) { c = tab + T * 16 + hh * 12 + 4 * (ch - 2); s = c + H * 12; }
    else { c = tab + T * 16 + H * 24 + w * 12 + 4 * (ch - 5); s = c + W * 12; }
    const uint4 raw = __ldg(src + i);
    uint32_t wds[4] = {raw.x, raw.y, raw.z, raw.w};
    float inv = 1.f, w8[8] = {1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f};
    if (nw) {  // uniform: every lane of a group is in the loop together
      inv = lc_rms_inv(lc_sumsq_lanes8(sumsq_chunk_bf16(wds), group), eps);
#pragma unroll
      for (int e = 0; e < 8; ++e) w8[e] = __ldg(nw + 8 * ch + e);
    }
    rot_chunk_bf16(wds, __ldg(reinterpret_cast<const float4 *>(c)),
                   __ldg(reinterpret_cast<const float4 *>(s)), nw != nullptr, inv, w8);
    dst[i] = make_uint4(wds[0], wds[1], wds[2], wds[3]);
  }
}

lc_status launch_rope_k(const void *src, void *dst, int batch, long long ntok, int heads,
                        int tok_offset, const lc_rope3d_s *rope, cudaStream_t stream,
                        const float *nw, float eps) {
  const long long n_chunks = (long long)batch * ntok * heads * (LC_HEAD_DIM / 8);
  int dev = 0, n_sm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  const long long want = (n_chunks + 255) / 256;
  const int grid = (int)(want < 8LL * n_sm ? want : 8LL * n_sm);
  rope_k_kernel<<<grid, 256, 0, stream>>>(static_cast<const uint4 *>(src),
                                          static_cast<uint4 *>(dst), n_chunks, heads, ntok,
                                          tok_offset, rope->tab, rope->T, rope->H, rope->W,
                                          lc_make_divmod(rope->H * rope->W),
                                          lc_make_divmod(rope->W), nw, eps);
  return lc_from_cuda(cudaGetLastError());
}

}  // namespace

lc_status lc_encode_segment(CUtensorMap *m, const void *base, int batch, long long ntot,
                            long long tok0, long long nseg, int heads) {
  return encode_segment(m, base, batch, ntot, tok0, nseg, heads);
}

lc_status lc_encode_f32_halfrows(CUtensorMap *m, const float *base, int batch, long long ntot,
                                 int heads) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return LC_ERR_CUDA;
  const long long row_bytes = (long long)heads * LC_HEAD_DIM * 4;
  cuuint64_t dims[4] = {LC_HEAD_DIM, (cuuint64_t)heads, (cuuint64_t)ntot, (cuuint64_t)batch};
  cuuint64_t strides[3] = {LC_HEAD_DIM * 4, (cuuint64_t)row_bytes, (cuuint64_t)(ntot * row_bytes)};
  cuuint32_t box[4] = {32, 1, 64, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<float *>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? LC_OK : LC_ERR_CUDA;
}

lc_status lc_rope_rows_bf16(const void *src, void *dst, int batch, long long ntok, int heads,
                            int tok_offset, const lc_rope3d_s *rope, const float *nw, float eps,
                            cudaStream_t stream) {
  if (ntok <= 0) return LC_OK;
  LC_CUDA_TRY(cudaStreamWaitEvent(stream, rope->ready, 0));
  return launch_rope_k(src, dst, batch, ntok, heads, tok_offset, rope, stream, nw, eps);
}

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

int *lc_noalloc_scratch_if_ready() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoallocMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  return g_noalloc_ptr[dev];
}

lc_status lc_launch_forward_sm100(const void *q, const void *k, const void *v, const void *cond_k,
                                  const void *cond_v, void *out, float *lse, int batch, int heads,
                                  float scale, lc_fwd_mode mode, bool cond_k_rotated,
                                  const lc_qk_norm &norm, const lc_bsa_plan_s *plan,
                                  const lc_rope3d_s *rope, int *dev_status, cudaStream_t stream,
                                  int *counter_scratch, const lc_shard_view *shard) {
  Sm100Params prm;
  memset(&prm, 0, sizeof(prm));
  const long long Nc = plan->Nc, Nn = plan->Nn, N = Nc + Nn;
  const bool cached = mode == LC_FWD_CACHED, cond_only = mode == LC_FWD_COND;
  const bool sharded = mode == LC_FWD_SHARD;
  if (counter_scratch && mode != LC_FWD_FULL) return LC_ERR_UNSUPPORTED;
  if (sharded != (shard != nullptr)) return LC_ERR_INVALID_ARGUMENT;
  if (cond_only && Nc == 0) return LC_OK;
  lc_status s = LC_OK;
  // Shard maps: per segment, the part of a shard buffer (tokens [lo, lo + n))
  // that lies in the segment; row_off[seg] = that part's first row counted
  // from the segment start (the kernel subtracts it from segment rows).
  const long long seg_lo[2] = {0, Nc}, seg_hi[2] = {Nc, N};
  auto encode_shard = [&](CUtensorMap *maps, const void *base, long long lo, long long n,
                          int *row_off) -> lc_status {
    bool have[2] = {false, false};
    for (int sg = 0; sg < 2; ++sg) {
      const long long a = lo > seg_lo[sg] ? lo : seg_lo[sg];
      const long long b = lo + n < seg_hi[sg] ? lo + n : seg_hi[sg];
      if (a >= b) continue;
      lc_status r = encode_segment(&maps[sg], base, batch, n, a - lo, b - a, heads);
      if (r != LC_OK) return r;
      if (row_off) row_off[sg] = (int)(a - seg_lo[sg]);
      have[sg] = true;
    }
    if (!have[0] && !have[1]) return LC_ERR_INVALID_ARGUMENT;
    if (!have[0]) maps[0] = maps[1];  // unused segment: a valid descriptor, never read
    if (!have[1]) maps[1] = maps[0];
    return LC_OK;
  };
  if (sharded) {
    s = encode_shard(prm.tmQ, q, shard->q_lo, shard->q_n, prm.q_row_off);
    if (s == LC_OK) s = encode_shard(prm.tmO, out, shard->q_lo, shard->q_n, nullptr);
    if (s == LC_OK) s = encode_shard(prm.tmK, k, shard->k_lo, shard->k_n, prm.k_row_off);
    if (s == LC_OK) s = encode_shard(prm.tmV, v, shard->k_lo, shard->k_n, nullptr);
    prm.lse_base[0] = (int)(seg_lo[0] - shard->q_lo);
    prm.lse_base[1] = (int)(seg_lo[1] - shard->q_lo);
    prm.lse_nq = (int)shard->q_n;
    prm.group_offset = 0;
    prm.n_groups_active = plan->G_active;  // groups with entries rank first
  } else if (cond_only) {  // condition queries over condition keys only
    s = encode_segment(&prm.tmQ[0], q, batch, Nc, 0, Nc, heads);
    if (s == LC_OK) s = encode_segment(&prm.tmO[0], out, batch, Nc, 0, Nc, heads);
    if (s == LC_OK) s = encode_segment(&prm.tmK[0], cond_k, batch, Nc, 0, Nc, heads);
    if (s == LC_OK) s = encode_segment(&prm.tmV[0], cond_v, batch, Nc, 0, Nc, heads);
    prm.lse_base[0] = 0;
    prm.lse_nq = (int)Nc;
    // grp_order ranks noisy groups first (every noisy list holds all Cb
    // condition blocks plus at least one noisy block, so it is longer than
    // any condition list); the condition groups are the last gc ranks.
    prm.group_offset = plan->gn;
    prm.n_groups_active = plan->gc;
  } else if (cached) {
    s = encode_segment(&prm.tmQ[1], q, batch, Nn, 0, Nn, heads);
    if (s == LC_OK) s = encode_segment(&prm.tmO[1], out, batch, Nn, 0, Nn, heads);
    if (s == LC_OK) s = encode_segment(&prm.tmK[1], k, batch, Nn, 0, Nn, heads);
    if (s == LC_OK) s = encode_segment(&prm.tmV[1], v, batch, Nn, 0, Nn, heads);
    if (s == LC_OK && Nc > 0) {
      s = encode_segment(&prm.tmK[0], cond_k, batch, Nc, 0, Nc, heads);
      if (s == LC_OK) s = encode_segment(&prm.tmV[0], cond_v, batch, Nc, 0, Nc, heads);
    }
    prm.lse_base[1] = 0;
    prm.lse_nq = (int)Nn;
    prm.group_offset = 0;
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
    prm.lse_base[0] = 0;
    prm.lse_base[1] = (int)Nc;
    prm.lse_nq = (int)N;
    prm.group_offset = 0;
    prm.n_groups_active = plan->G;
  }
  if (s != LC_OK) return s;
  if (sharded) {
    // encode_shard filled every map
  } else if (cond_only) {  // keep the unused noisy maps valid descriptors
    prm.tmQ[1] = prm.tmQ[0]; prm.tmK[1] = prm.tmK[0];
    prm.tmV[1] = prm.tmV[0]; prm.tmO[1] = prm.tmO[0];
  } else if (Nc == 0) {  // keep the unused condition maps valid descriptors
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
  prm.n_groups = plan->G;
  prm.n_blocks = plan->Cb + plan->Nb;
  prm.ent_cap = (int)plan->nnz;
  prm.k_prerotated = 0;
  prm.q_norm_w = norm.q_w;
  prm.k_norm_w = norm.k_w;
  prm.norm_eps = norm.eps;
  long long total = (long long)batch * heads * prm.n_groups_active;
  if (total == 0) return LC_OK;
  if (total >= (1LL << 31)) return LC_ERR_UNSUPPORTED;
  prm.total_items = (int)total;
  prm.tab_floats = (int)rope->n_floats;
  prm.scale_log2 = scale * 1.4426950408889634f;

  const size_t smem = 1024 + SmemOffsets::tab + sizeof(float) * (size_t)rope->n_floats;
  if (smem > 227 * 1024) return LC_ERR_UNSUPPORTED;
  // The kernel's setmaxnreg split needs at least kRegsAtLaunchMin registers
  // per thread at launch; with fewer, raising the softmax warps' count could
  // never complete, so such a build is refused instead of launched.
  const bool with_norm = prm.q_norm_w || prm.k_norm_w;
  void (*const kern)(const Sm100Params) = with_norm ? bsa_sm100_kernel<true>
                                                    : bsa_sm100_kernel<false>;
  static int regs_at_launch[2] = {-1, -1};
  int &regs = regs_at_launch[with_norm ? 1 : 0];
  if (regs < 0) {
    cudaFuncAttributes fa;
    LC_CUDA_TRY(cudaFuncGetAttributes(&fa, kern));
    regs = fa.numRegs;
  }
  if (regs < kRegsAtLaunchMin) return LC_ERR_UNSUPPORTED;
  LC_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  int dev = 0, n_sm = 0;
  LC_CUDA_TRY(cudaGetDevice(&dev));
  LC_CUDA_TRY(cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev));
  const int grid = (int)(total < n_sm ? total : n_sm);

  if (counter_scratch) {  // caller-provided scratch: nothing is allocated
    prm.work_counter = counter_scratch;
    cudaError_t e = cudaMemsetAsync(counter_scratch, 0, sizeof(int), stream);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(stream, plan->ready, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(stream, rope->ready, 0);
    if (e == cudaSuccess) {
      kern<<<grid, kThreads, smem, stream>>>(prm);
      e = cudaGetLastError();
    }
    return lc_from_cuda(e);
  }
  // K is rotated once per call into scratch (one pass over K) and the kernel
  // loads it rotated; rotating every loaded K tile in the kernel instead (as
  // the allocation-free entry point does, having no scratch) measured slower.
  // (A shard whose K arrives rotated needs no prepass.)
  const bool k_prepass = !(sharded && shard->k_rotated);
  if (sharded && shard->k_rotated) prm.k_prerotated = 1;
  if (sharded && shard->q_rotated) prm.q_prerotated = 1;
  int *counter = nullptr;
  void *k_rot = nullptr, *ck_rot = nullptr;
  cudaMemPool_t pool = lc_scratch_pool(&s);
  if (s != LC_OK) return s;
  cudaError_t e = cudaStreamWaitEvent(stream, rope->ready, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(stream, plan->ready, 0);
  if (e == cudaSuccess && k_prepass) {
    // K of the query-side tensor (all tokens, the noisy ones, or the shard's).
    if (!cond_only) {
      const long long kn = sharded ? shard->k_n : (cached ? Nn : N);
      const int k_tok0 = sharded ? (int)shard->k_lo : (cached ? (int)Nc : 0);
      e = cudaMallocFromPoolAsync(&k_rot, (size_t)batch * kn * heads * LC_HEAD_DIM * 2, pool,
                                  stream);
      if (e == cudaSuccess)
        s = launch_rope_k(k, k_rot, batch, kn, heads, k_tok0, rope, stream, norm.k_w, norm.eps);
    }
    // Separately supplied condition K, unless the caller rotated it already.
    if (e == cudaSuccess && s == LC_OK && (cached || cond_only) && Nc > 0 && !cond_k_rotated) {
      e = cudaMallocFromPoolAsync(&ck_rot, (size_t)batch * Nc * heads * LC_HEAD_DIM * 2, pool,
                                  stream);
      if (e == cudaSuccess)
        s = launch_rope_k(cond_k, ck_rot, batch, Nc, heads, 0, rope, stream, norm.k_w, norm.eps);
    }
    if (e == cudaSuccess && s == LC_OK) {
      if (ck_rot) s = encode_segment(&prm.tmK[0], ck_rot, batch, Nc, 0, Nc, heads);
      if (sharded) {
        s = encode_shard(prm.tmK, k_rot, shard->k_lo, shard->k_n, prm.k_row_off);
      } else if (cond_only) {
        prm.tmK[1] = prm.tmK[0];
      } else if (cached) {
        if (s == LC_OK) s = encode_segment(&prm.tmK[1], k_rot, batch, Nn, 0, Nn, heads);
        if (s == LC_OK && Nc == 0) prm.tmK[0] = prm.tmK[1];
      } else {
        s = encode_segment(&prm.tmK[1], k_rot, batch, N, Nc, Nn, heads);
        if (s == LC_OK && Nc > 0) s = encode_segment(&prm.tmK[0], k_rot, batch, N, 0, Nc, heads);
        if (s == LC_OK && Nc == 0) prm.tmK[0] = prm.tmK[1];
      }
      prm.k_prerotated = 1;
    }
  }
  const bool overlap = sharded && shard->overlap_previous;
  if (overlap && e == cudaSuccess && s == LC_OK) {
    // The plan's own scheduler (zero between launches) and a programmatic
    // dependent launch: no stream operation separates it from the previous kernel.
    prm.work_counter = plan->sched;
    prm.exit_counter = plan->sched + 1;
    prm.pdl = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, prm);
  } else {
    if (e == cudaSuccess && s == LC_OK)
      e = cudaMallocFromPoolAsync(reinterpret_cast<void **>(&counter), sizeof(int), pool, stream);
    if (e == cudaSuccess && s == LC_OK) {
      prm.work_counter = counter;
      e = cudaMemsetAsync(counter, 0, sizeof(int), stream);
      if (e == cudaSuccess) {
        kern<<<grid, kThreads, smem, stream>>>(prm);
        e = cudaGetLastError();
      }
    }
  }
  if (counter) cudaFreeAsync(counter, stream);
  if (k_rot) cudaFreeAsync(k_rot, stream);
  if (ck_rot) cudaFreeAsync(ck_rot, stream);
  if (s != LC_OK) return s;
  return lc_from_cuda(e);
}

lc_status lc_launch_watchdog_selftest(int *dev_status, long long timeout_ns, cudaStream_t stream) {
  watchdog_selftest_kernel<<<1, 32, 0, stream>>>(dev_status, timeout_ns);
  LC_CUDA_TRY(cudaGetLastError());
  return LC_OK;
}
