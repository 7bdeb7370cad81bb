// fa_fwd.cu -- FlashAttention forward for NVIDIA B200 (sm_100a) and its C ABI.
//
// What is computed (the method of the pages, restated):
//   O = softmax(scale * Q K^T [+ causal mask]) V per (batch, head), and the
//   natural-log log-sum-exp of every row.  The key axis is walked tile by
//   tile with an online softmax -- a running row max m and a running exp-sum
//   l, both rescaled whenever m grows, with the partial output rescaled the
//   same way -- so the score matrix never leaves the chip.
//   Page "FlashAttention: long-text inference without running out of memory"
//   (ai6s.net/6a0d42d8), section "FlashAttention's answer: tiling + online
//   normalisation" (the m / l recurrence); page "catlass FlashAttention
//   template tuning" (hwcomputing.csdn.net/6a0d4681), section "causal mask
//   implementations", mode 2 (skip key tiles above the diagonal, mask inside
//   diagonal tiles); page "64K long-sequence FlashAttention"
//   (ai6s.net/6a140d07), section "layer 2: numerical stability" (the per-row
//   LSE) and section "multi-AI-Core load balancing" (balanced scheduling of
//   uneven tile counts).
//
// How it maps onto sm_100a (a design of its own, not the pages' Ascend one):
//   * One persistent CTA per SM (10 warps, 320 threads).  A work unit is two
//     128-row query tiles of one (batch, head); units are walked longest
//     first inside L2-sized groups of heads (static schedule, no workspace).
//   * Warp 8 (load): TMA loads of Q tiles and a ring of K / V tiles
//     (128 keys x D, 128-byte swizzle) behind full / empty mbarriers.
//   * Warp 9 (MMA): one thread issues tcgen05.mma.  S_t = Q_t K^T goes to
//     tensor memory (fp32, 128 lanes x 128 columns); O_t += P_t V reads P_t
//     from tensor memory (it overwrites the first 64 columns of S_t) and V
//     from shared memory.  TMEM: S0 | S1 | O0 | O1 = 512 columns.
//   * Warps 0-3 / 4-7 (softmax warpgroups, one per query tile): each thread
//     owns one query row.  It reads its S row from TMEM, masks it (diagonal
//     and ragged-tail tiles only), updates m and l in the exp2 domain with
//     the scale folded in (scale * log2 e), writes P (fp16 / bf16) back to
//     TMEM, rescales its O row when m grew, and at the end normalises O by l,
//     stages it in shared memory (swizzled) and TMA-stores it, and writes LSE.
//   * The two query tiles ping-pong: while one warpgroup computes its
//     softmax the tensor core works on the other tile.
//   * Every mbarrier wait is bounded (globaltimer); a wait that runs past the
//     limit sets a device error word, the CTA drains its copies and MMAs,
//     frees TMEM and returns.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "fa_fwd.h"

#define FA_VERSION 10000

namespace fa {

// ----------------------------------------------------------------------------- constants

constexpr int BM = 128;             // query rows per tile (one TMEM lane per row)
constexpr int BN = 128;             // keys per K / V tile
constexpr int NQ = 2;               // query tiles per work unit (ping-pong)
constexpr int UNIT_ROWS = NQ * BM;  // 256
constexpr int NUM_THREADS = 384;    // warps 0-7 softmax, 8 load, 9 MMA, 10-11 idle (producer warpgroup)
// Register split (setmaxnreg): the launch gives 384 x 168 = 64512 registers;
// the producer warpgroup drops to 112 per thread and the two softmax
// warpgroups rise to 184: 128 x 112 + 256 x 184 = 61440, within the launch.
constexpr int REGS_PRODUCER = 112;
constexpr int REGS_SOFTMAX = 184;
static_assert(128 * REGS_PRODUCER + 256 * REGS_SOFTMAX <= NUM_THREADS * 168, "register split exceeds the launch");
constexpr int LOAD_WARP = 8;
constexpr int MMA_WARP = 9;
constexpr int TMEM_COLS = 512;
constexpr int BOX_BYTES = BM * 128;  // one 128-row x 64-element (128-byte) TMA box
constexpr int UQ_DEPTH = 4;           // unit ids in flight between the producer and the consumers
constexpr int UQ_CONSUMERS = 9;       // arrivals that free a unit-id slot: the MMA warp + 8 softmax warps
// Defaults of the lazy rescale (fa_fwd_options): O / l are rescaled only when
// a row max grows by more than the threshold (log2 units), and for bf16 a
// moved reference sits the headroom above the tile max.
constexpr float RESCALE_LOG2_DEFAULT = 15.0f;
constexpr float HEADROOM_LOG2_DEFAULT = 8.0f;
#ifndef FA_EMU_PAIRS
#define FA_EMU_PAIRS 0
#endif
// Of the 64 exp2 pairs of a 128-key row, this many (spread evenly) run on the
// FMA pipe.  The softmax loop is bound by latency and instruction dispatch as
// much as by MUFU: a MUFU pair costs 1 dispatch slot per value but 8 pipe
// cycles, an emulated pair about 22 dispatch slots.  Measured on the four
// large workloads (calls of the variants interleaved, sustained clocks), 4 to
// 10 of 64 are 3-10 % slower than none, so the default is 0.
constexpr int EMU_PAIRS = FA_EMU_PAIRS;
__host__ __device__ constexpr bool emulated_pair(int i, int e) { return (i * e) / 64 != ((i + 1) * e) / 64; }

template <int D>
struct Cfg {
  static constexpr int TILE_BYTES = BM * D * 2;             // one Q / K / V / O tile
  static constexpr int NSLOT = (D == 128) ? 5 : 8;           // K / V ring slots
  static constexpr int NBOX = D / 64;                        // 128-byte boxes per row
  // mbarrier indices
  static constexpr int KV_FULL = 0;
  static constexpr int KV_EMPTY = NSLOT;
  static constexpr int Q_FULL = 2 * NSLOT;
  static constexpr int Q_EMPTY = Q_FULL + NQ;
  static constexpr int S_FULL = Q_EMPTY + NQ;
  static constexpr int P_FULL = S_FULL + NQ;
  static constexpr int O_FULL = P_FULL + NQ;
  static constexpr int O_EMPTY = O_FULL + NQ;
  static constexpr int EPI = O_EMPTY + NQ;
  static constexpr int DRAIN = EPI + NQ;
  static constexpr int UQ_FULL = DRAIN + 1;     // unit-id ring: producer -> MMA warp and softmax warps
  static constexpr int UQ_EMPTY = UQ_FULL + UQ_DEPTH;
  static constexpr int NBAR = UQ_EMPTY + UQ_DEPTH;
  static constexpr int SMEM_Q = 0;
  static constexpr int SMEM_KV = NQ * TILE_BYTES;
  static constexpr int SMEM_BAR = SMEM_KV + NSLOT * TILE_BYTES;
  static constexpr int SMEM_MISC = SMEM_BAR + NBAR * 8;       // tmem address, abort flag, unit-id ring
  static constexpr int SMEM_BYTES = SMEM_MISC + 8 + 4 * UQ_DEPTH + 1024;  // + slack for 1024-byte alignment
};

struct Params {
  float* lse;
  unsigned int* sched;  // work counter for the dynamic schedule (zeroed before launch), or nullptr: static
  int B, H, Sq, Sk;      // variable-length batch: Sq, Sk = the longest sequence
  int nqb;             // query units per head: ceil(Sq / 256)
  int tk;              // key tiles: ceil(Sk / 128)
  int bh;              // heads this launch computes (B * H, or a range of them)
  int head0;           // first head of the range: flattened index b * H + h
  int group_heads;     // heads per L2 group of the schedule
  int total_units;     // bh * nqb
  int causal;
  int bhsd;            // 1: [B,H,S,D], 0: [B,S,H,D]
  float scale_log2;    // scale * log2(e)
  unsigned long long wait_limit_ns;
  int withhold_loads;  // self-test of the bounded waits: the producer issues no loads
  // Variable-length batch (packed [total, H, D] rows), else cu_q == nullptr:
  // sequence b has query rows [cu_q[b], cu_q[b+1]) and keys [cu_k[b], cu_k[b+1]).
  const int* cu_q;
  const int* cu_k;
  int total_q, total_k;
  uint8_t* o;           // O base (packed and ring-step launches store each row directly)
  long long o_bs, o_hs, o_rs;  // element offsets in O of a batch, a head and a row (row stores)
  long long lse_bs, lse_hs;   // LSE offsets of a batch and of a head (plus the row)
  // Ring step: nseg (1 or 2) query segments with disjoint rows, segment 0's
  // units first (seg_units0 of them).  Segment s takes query rows
  // [seg_row0[s], seg_row0[s] + Sq) of Q / O / LSE and keys
  // [seg_key0[s], seg_key0[s] + seg_sk[s]) of K / V; with seg_causal[s], key c
  // of the segment is visible from its row r iff c <= r + seg_coff[s].
  // seg_flags[s]: bit 0 (first) no earlier result to merge, bit 1 (last) the
  // merged result is final (O in the input dtype); otherwise it is the running
  // result: fp32 O in acc (strides of O) and its LSE in lse.
  int nseg, seg_units0;
  int seg_row0[2], seg_key0[2], seg_sk[2], seg_coff[2], seg_causal[2], seg_flags[2];
  float* acc;
  // Split-KV (a ring-step launch with split_n > 0 instead of segments): split
  // s takes keys [s * split_keys, (s + 1) * split_keys) of every query row
  // (no mask) and writes its own result as the rows' first, not last, one:
  // fp32 O to rows s * Sq + r of acc and its LSE to the same rows of lse;
  // units of split s are [s * seg_units0, (s + 1) * seg_units0).
  int split_n, split_keys;
  // Lazy rescale: the reference max moves only when a tile's max exceeds it
  // by more than rescale_log2 (weights against a stale reference stay below
  // rescale_pow2 = 2^rescale_log2); bf16 sets a moved reference headroom_log2
  // above the tile max.
  float rescale_log2, rescale_pow2, headroom_log2;
  // Optional statistics (nullptr: off), per warp and key tile after a unit's
  // first: [0] such warp-tiles, [1] speculative pass rejected (exact
  // recompute), [2] O rescaled, [3] accepted with a weight above half the
  // bound (a stale reference close to its limit).
  unsigned long long* counts;
};

// Device error word: bit 0 a wait ran out (FA_ERR_TIMEOUT), bit 1 invalid
// sequence offsets of a variable-length batch (FA_ERR_INVALID_ARG).
__device__ int g_dev_error = 0;


// ----------------------------------------------------------------------------- PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase of the given parity.  Returns false (for the
// whole warp) if the CTA was aborted or the limit ran out; the first warp to
// run out records the timeout in the device error word.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         uint64_t limit_ns) {
  bool ok = mbar_try_wait(bar, parity);
  if (!ok) {
    const uint64_t t0 = globaltimer_ns();
    while (true) {
#pragma unroll 1
      for (int i = 0; i < 16 && !ok; ++i) ok = mbar_try_wait(bar, parity);
      if (ok) break;
      if (*abort_flag) break;
      if (globaltimer_ns() - t0 > limit_ns) {
        *abort_flag = 1;
        atomicOr(&g_dev_error, 1);
        break;
      }
    }
  }
  return __all_sync(0xffffffffu, ok);
}

// Bounded wait for one thread (the producer and MMA roles run on lane 0 only).
__device__ __forceinline__ bool wait_bar1(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 16; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      atomicOr(&g_dev_error, 1);
      return false;
    }
  }
}

// Bounded wait used only while draining (ignores the abort flag).
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > limit_ns) {
      atomicOr(&g_dev_error, 1);
      return;
    }
  }
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
      : "memory");
}

// The same load with an L2 cache policy (createpolicy): evict_last for data
// that later loads read again, evict_first for data read once.
__device__ __forceinline__ void tma_load_4d_hint(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1,
                                                 int c2, int c3, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, uint32_t src, int c0, int c1,
                                             int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

__device__ __forceinline__ void tma_store_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void tma_store_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void tma_store_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// tcgen05 -------------------------------------------------------------------

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// One lane of a converged warp: the lane that issues a group of tcgen05.mma.
// The *_elect forms below are executed by a whole (converged) warp, so their
// operands stay warp-uniform; one elected lane issues the instruction.
__device__ __forceinline__ bool elect_one() {
  uint32_t e;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "elect.sync _|p, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(e));
  return e != 0;
}

__device__ __forceinline__ void tc_commit_elect(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(bar)
      : "memory");
}

// D(tmem) (+)= A(smem desc) * B(smem desc)
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D(tmem) (+)= A(tmem) * B(smem desc)
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 32 columns of 32-bit words: thread i of the warp gets lane
// (warp quadrant * 32 + i), columns [col, col + 32).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
      "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]),
      "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]),
      "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Keeps every use of r after the preceding tcgen05.wait::ld (both are volatile asm).
template <int N>
__device__ __forceinline__ void reg_fence(uint32_t (&r)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

// Columns [col, col + 32 * N) of this warp's 32 lanes into r, one wait for all.
template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[32 * N]) {
#pragma unroll
  for (int c = 0; c < N; ++c) tmem_ld32(taddr + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&r[32 * c]));
  tmem_wait_ld();
  reg_fence(r);
}

__device__ __forceinline__ void prefetch_l2(const void* ptr) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(ptr));
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  if constexpr (BF16) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  } else {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
}

template <bool BF16>
__device__ __forceinline__ float round_to_input(float x) {
  if constexpr (BF16) return __bfloat162float(__float2bfloat16_rn(x));
  else return __half2float(__float2half_rn(x));
}

// Packed fp32 pairs (sm_100 f32x2 arithmetic: one instruction for two lanes of work).
__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
  uint64_t d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
  return d;
}
__device__ __forceinline__ void f2unpack(uint64_t d, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(d));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ uint32_t imad_shl23(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mad.lo.u32 %0, %1, 8388608, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint64_t fsub2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// 2^x for two values on the FMA pipe instead of MUFU.  x = j + r with
// j = round(x): adding 1.5 * 2^23 leaves j in the low mantissa bits, so
// (x + 1.5 * 2^23) - 1.5 * 2^23 = j exactly and r = x - j lies in [-1/2, 1/2].
// 2^r is a polynomial (constant term 1; near-minimax in relative error, fitted
// by csrc/gen_exp2_poly.py: 1.0e-4 at degree 3, 2.9e-6 at degree 4), and 2^j
// is added to its exponent field.  x is clamped to [-127, 64]: at -127, r = 0
// and the polynomial is exactly 1, whose exponent field 127 the addition
// takes to zero, so -inf (a masked key) and anything below give exactly +0;
// just above -127 the result is a denormal below 2^-126 (negligible beside
// the row's largest weight, at least 2^-headroom); an argument above 64
// (only possible on a rejected speculative pass, see the softmax) still gives
// a large positive value.
template <int DEG>
__device__ __forceinline__ void exp2_poly_pair(uint64_t x2, float& y0, float& y1) {
  float xin0, xin1;
  f2unpack(x2, xin0, xin1);
  const uint64_t x = f2pack(fminf(fmaxf(xin0, -127.f), 64.f), fminf(fmaxf(xin1, -127.f), 64.f));
  const uint64_t magic = f2pack(12582912.f, 12582912.f);
  const uint64_t t = fadd2(x, magic);
  const uint64_t r = fsub2(x, fsub2(t, magic));
  uint64_t p;
  if constexpr (DEG == 3) {
    p = ffma2(r, f2pack(5.500874668e-02f, 5.500874668e-02f), f2pack(2.422107607e-01f, 2.422107607e-01f));
    p = ffma2(p, r, f2pack(6.932829022e-01f, 6.932829022e-01f));
  } else {
    p = ffma2(r, f2pack(9.582836181e-03f, 9.582836181e-03f), f2pack(5.590641499e-02f, 5.590641499e-02f));
    p = ffma2(p, r, f2pack(2.402409911e-01f, 2.402409911e-01f));
    p = ffma2(p, r, f2pack(6.931241751e-01f, 6.931241751e-01f));
  }
  p = ffma2(p, r, f2pack(1.f, 1.f));
  float p0, p1, t0, t1;
  f2unpack(p, p0, p1);
  f2unpack(t, t0, t1);
  // 2^j into the exponent field: bits(t) * 2^23 + bits(p) (an integer multiply-add,
  // which runs on the FMA pipe); bits(t) * 2^23 keeps only j * 2^23 modulo 2^32
  y0 = __uint_as_float(imad_shl23(__float_as_uint(t0), __float_as_uint(p0)));
  y1 = __uint_as_float(imad_shl23(__float_as_uint(t1), __float_as_uint(p1)));
}

// max over the row of s * c (c > 0: max(s) * c; c < 0: min(s) * c; c = 0: 0).
__device__ __forceinline__ float row_max_scaled(const uint32_t (&sr)[BN], float c) {
  float a[4];
  if (c >= 0.f) {
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      a[g] = __uint_as_float(sr[32 * g]);
#pragma unroll
      for (int e = 1; e < 31; e += 2)
        a[g] = max3f(a[g], __uint_as_float(sr[32 * g + e]), __uint_as_float(sr[32 * g + e + 1]));
      a[g] = fmaxf(a[g], __uint_as_float(sr[32 * g + 31]));
    }
    return max3f(a[0], a[1], fmaxf(a[2], a[3])) * c;
  }
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    a[g] = __uint_as_float(sr[32 * g]);
#pragma unroll
    for (int e = 1; e < 32; ++e) a[g] = fminf(a[g], __uint_as_float(sr[32 * g + e]));
  }
  return fminf(fminf(a[0], a[1]), fminf(a[2], a[3])) * c;
}

// P = 2^(s * cc + neg_m) for the row: EMU of the 64 pairs (spread evenly) on
// the FMA pipe, the rest on MUFU; packed to the input dtype into pk (two per 32-bit word).
// Returns the fp32 row sum; ymax gets the largest fp32 weight (the one the
// rounding correction is taken from, and the speculation check).
template <bool BF16, int EMU>
__device__ __forceinline__ float exp_pack_row(const uint32_t (&sr)[BN], float cc, float neg_m, uint32_t (&pk)[BN / 2],
                                              float& ymax) {
  const uint64_t cc2 = f2pack(cc, cc), nm2 = f2pack(neg_m, neg_m);
  uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
  float mx[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < BN / 2; ++i) {
    const uint64_t x2 = ffma2(f2pack(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])), cc2, nm2);
    float y0, y1;
    if (emulated_pair(i, EMU)) {
      exp2_poly_pair<BF16 ? 3 : 4>(x2, y0, y1);
    } else {
      float x0, x1;
      f2unpack(x2, x0, x1);
      y0 = ex2(x0);
      y1 = ex2(x1);
    }
    acc[i & 3] = fadd2(acc[i & 3], f2pack(y0, y1));
    mx[i & 7] = max3f(mx[i & 7], y0, y1);
    pk[i] = pack2<BF16>(y0, y1);
  }
  ymax = max3f(max3f(mx[0], mx[1], mx[2]), max3f(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
  float a0, a1;
  f2unpack(fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3])), a0, a1);
  return a0 + a1;
}

// ----------------------------------------------------------------------------- descriptors

// Shared-memory matrix descriptor (sm_100 format): start, leading and stride
// byte offsets (>> 4), version 1 at bit 46, 128-byte swizzle (2) at bits 61-63.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor, kind::f16: fp32 accumulator, A and B of the same
// 16-bit type (0 fp16, 1 bf16), A K-major, B K-major (0) or MN-major (1).
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, uint32_t fmt, uint32_t b_mn_major) {
  return (1u << 4) | (fmt << 7) | (fmt << 10) | (b_mn_major << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// ----------------------------------------------------------------------------- schedule

// Launch kinds (the kernel's KIND): a dense batch, a packed variable-length
// batch, a ring step (query segments merged into a running result).
constexpr int DENSE = 0, PACKED = 1, RING = 2;

struct Unit {
  int b, h, r0;     // batch, head, first query row of the unit (within its sequence)
  int causal, coff; // causal mask (key c visible from row r iff c <= r + coff)
  int seg;          // ring-step segment (or split)
  int ob;           // first row of the unit's results in O / LSE (ring step and split-KV)
  int rows[NQ];     // valid rows of each query tile
  int n[NQ];        // key tiles each query tile visits (0: tile inactive)
  int sq, sk;       // the sequence's query and key lengths
  int rb, kb;       // its first query row and key row in the tensors (0 for a dense batch)
  int tb;           // batch coordinate of the tensor maps (0 for a packed batch)
};

// Units are grouped by heads so that the K / V of a group stay in L2; inside
// a group the longest units (causal: the last query rows) come first.
template <int KIND>
__device__ __forceinline__ Unit decode_unit(const Params& p, int u) {
  Unit un;
  un.causal = p.causal;
  un.coff = 0;
  un.seg = 0;
  if constexpr (KIND == RING) {
    // (selects rather than indexing: a dynamic index into the parameters
    // would copy them to local memory)
    if (p.split_n > 0) {
      un.seg = u / p.seg_units0;
      u -= un.seg * p.seg_units0;
      un.causal = 0;
    } else {
      un.seg = u >= p.seg_units0 ? 1 : 0;
      if (un.seg) u -= p.seg_units0;
      un.causal = un.seg ? p.seg_causal[1] : p.seg_causal[0];
      un.coff = un.seg ? p.seg_coff[1] : p.seg_coff[0];
    }
  }
  const int per_group = p.group_heads * p.nqb;
  const int g = u / per_group;
  const int r = u - g * per_group;
  const int gs = min(p.group_heads, p.bh - g * p.group_heads);
  const int level = r / gs;
  const int bh = p.head0 + g * p.group_heads + (r - level * gs);
  const int qblk = un.causal ? (p.nqb - 1 - level) : level;
  un.b = bh / p.H;
  un.h = bh - un.b * p.H;
  un.r0 = qblk * UNIT_ROWS;
  if constexpr (KIND == PACKED) {
    // Every role decodes the same offsets.  Offsets that cannot describe a
    // sequence of this batch (and a sequence with queries but no keys) make
    // the unit empty and are reported in the device error word.
    const int q0 = p.cu_q[un.b], q1 = p.cu_q[un.b + 1], k0 = p.cu_k[un.b], k1 = p.cu_k[un.b + 1];
    const bool bad = q0 < 0 || q1 < q0 || q1 > p.total_q || q1 - q0 > p.Sq || k0 < 0 || k1 < k0 ||
                     k1 > p.total_k || k1 - k0 > p.Sk || (k1 == k0 && q1 > q0);
    if (bad && un.r0 == 0) atomicOr(&g_dev_error, 2);
    un.sq = bad ? 0 : q1 - q0;
    un.sk = bad ? 0 : k1 - k0;
    un.rb = q0;
    un.kb = k0;
    un.tb = 0;
    un.ob = q0;
  } else if constexpr (KIND == RING) {
    un.sq = p.Sq;
    un.tb = un.b;
    if (p.split_n > 0) {
      un.kb = un.seg * p.split_keys;
      un.sk = min(p.split_keys, p.Sk - un.kb);
      un.rb = 0;
      un.ob = un.seg * p.Sq;
    } else {
      un.sk = un.seg ? p.seg_sk[1] : p.seg_sk[0];
      un.rb = un.seg ? p.seg_row0[1] : p.seg_row0[0];
      un.kb = un.seg ? p.seg_key0[1] : p.seg_key0[0];
      un.ob = un.rb;
    }
  } else {
    un.sq = p.Sq;
    un.sk = p.Sk;
    un.rb = 0;
    un.kb = 0;
    un.tb = un.b;
    un.ob = 0;
  }
#pragma unroll
  for (int t = 0; t < NQ; ++t) {
    const int first = un.r0 + t * BM;
    const int rows = max(0, min(BM, un.sq - first));
    un.rows[t] = rows;
    if (rows == 0) {
      un.n[t] = 0;
    } else if (un.causal) {
      const int last_key = min(first + rows - 1 + un.coff, un.sk - 1);
      un.n[t] = last_key / BN + 1;
    } else {
      un.n[t] = (un.sk + BN - 1) / BN;
    }
  }
  return un;
}

// ----------------------------------------------------------------------------- kernel

template <int D, bool BF16, int KIND>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    fa_fwd_kernel(const __grid_constant__ Params p, const __grid_constant__ CUtensorMap tmQ,
                  const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ CUtensorMap tmO) {
  using C = Cfg<D>;
  // Packed and ring-step launches store O row by row from registers (a tile
  // may end inside a sequence or a segment, where a TMA store would also
  // write the next one's rows), so Q is released after its last read.
  constexpr bool ROWSTORE = KIND != DENSE;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sQ = smem_u32(smem + C::SMEM_Q);
  const uint32_t sKV = smem_u32(smem + C::SMEM_KV);
  const uint32_t bars = smem_u32(smem + C::SMEM_BAR);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::SMEM_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::SMEM_MISC + 4);
  volatile int* uq_ids = reinterpret_cast<volatile int*>(smem + C::SMEM_MISC + 8);
  auto bar = [&](int i) -> uint32_t { return bars + 8u * (uint32_t)i; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint64_t limit = p.wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NSLOT; ++s) {
      mbar_init(bar(C::KV_FULL + s), 1);
      mbar_init(bar(C::KV_EMPTY + s), 1);
    }
    for (int t = 0; t < NQ; ++t) {
      mbar_init(bar(C::Q_FULL + t), 1);
      mbar_init(bar(C::Q_EMPTY + t), 1);
      mbar_init(bar(C::S_FULL + t), 1);
      mbar_init(bar(C::P_FULL + t), BM / 32);   // one arrival per softmax warp
      mbar_init(bar(C::O_FULL + t), 1);
      mbar_init(bar(C::O_EMPTY + t), BM / 32);
      mbar_init(bar(C::EPI + t), BM);
    }
    mbar_init(bar(C::DRAIN), 1);
    for (int i = 0; i < UQ_DEPTH; ++i) {
      mbar_init(bar(C::UQ_FULL + i), 1);
      mbar_init(bar(C::UQ_EMPTY + i), UQ_CONSUMERS);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == MMA_WARP) {
    tmem_alloc(smem_u32(tmem_holder), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  constexpr uint32_t FMT = BF16 ? 1u : 0u;
  constexpr uint32_t IDESC_QK = idesc_f16(BM, BN, FMT, 0);
  constexpr uint32_t IDESC_PV = idesc_f16(BM, D, FMT, 1);

  if (warp >= LOAD_WARP) {
   asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REGS_PRODUCER));
   if (warp == LOAD_WARP) {
    // ------------------------------------------------------------------ TMA producer (lane 0)
    if (lane == 0) {
      uint32_t kv_cnt = 0;
      uint32_t q_use[NQ] = {0, 0};
      bool ok = true;
      // Work units: the first is blockIdx.x; later ones come from the work
      // counter (dynamic schedule: units handed out in longest-first order)
      // or every gridDim.x-th unit (static schedule).  Each id, and finally an
      // end-of-work id, is passed to the MMA warp and the softmax warps
      // through the unit-id ring.
      int u = blockIdx.x;
      uint32_t uq_pos = 0;
      while (ok) {
        const uint32_t qs = uq_pos % UQ_DEPTH;
        ok = wait_bar1(bar(C::UQ_EMPTY + qs), ((uq_pos / UQ_DEPTH) & 1u) ^ 1u, abort_flag, limit);
        if (!ok) break;
        uq_ids[qs] = u;
        mbar_arrive(bar(C::UQ_FULL + qs));
        ++uq_pos;
        if (u >= p.total_units) break;
        if (p.withhold_loads) {
          // Self-test: nothing is loaded, so every consumer's wait for Q or
          // K / V runs out, and nothing is in flight when the CTA drains.
          u += (int)gridDim.x;
          continue;
        }
        const Unit un = decode_unit<KIND>(p, u);
        const int n = max(un.n[0], un.n[1]);
#pragma unroll
        for (int t = 0; t < NQ; ++t) {
          if (un.n[t] == 0 || !ok) continue;
          ok = wait_bar1(bar(C::Q_EMPTY + t), (q_use[t] & 1u) ^ 1u, abort_flag, limit);
          if (!ok) break;
          ++q_use[t];
          mbar_arrive_expect_tx(bar(C::Q_FULL + t), C::TILE_BYTES);
          const int s0 = un.rb + un.r0 + t * BM;
          for (int bx = 0; bx < C::NBOX; ++bx)
            tma_load_4d(sQ + t * C::TILE_BYTES + bx * BOX_BYTES, &tmQ, bar(C::Q_FULL + t), bx * 64,
                        p.bhsd ? s0 : un.h, p.bhsd ? un.h : s0, un.tb);
        }
        for (int j = 0; j < n && ok; ++j) {
          for (int kv = 0; kv < 2; ++kv) {
            const uint32_t slot = kv_cnt % C::NSLOT;
            const uint32_t use = kv_cnt / C::NSLOT;
            ok = wait_bar1(bar(C::KV_EMPTY + slot), (use & 1u) ^ 1u, abort_flag, limit);
            if (!ok) break;
            mbar_arrive_expect_tx(bar(C::KV_FULL + slot), C::TILE_BYTES);
            const CUtensorMap* map = kv ? &tmV : &tmK;
            const int s0 = un.kb + j * BN;
            for (int bx = 0; bx < C::NBOX; ++bx)
              tma_load_4d(sKV + slot * C::TILE_BYTES + bx * BOX_BYTES, map, bar(C::KV_FULL + slot),
                          bx * 64, p.bhsd ? s0 : un.h, p.bhsd ? un.h : s0, un.tb);
            ++kv_cnt;
          }
        }
        // The next unit is claimed only now, once every load of this one is
        // issued: the CTA then gets work about when it can start on it, which
        // keeps the longest-first hand-out balanced.
        u = p.sched ? (int)(gridDim.x + atomicAdd(p.sched, 1u)) : u + (int)gridDim.x;
      }
      // Drain: wait until every load this thread issued has landed.
      const uint32_t first = kv_cnt > (uint32_t)C::NSLOT ? kv_cnt - C::NSLOT : 0u;
      for (uint32_t c = first; c < kv_cnt; ++c)
        drain_wait(bar(C::KV_FULL + c % C::NSLOT), (c / C::NSLOT) & 1u, limit);
#pragma unroll
      for (int t = 0; t < NQ; ++t)
        if (q_use[t]) drain_wait(bar(C::Q_FULL + t), (q_use[t] - 1) & 1u, limit);
    }
    __syncwarp();
  } else if (warp == MMA_WARP) {
    // ------------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop in step (warp-uniform waits and
    // descriptors); each tcgen05 instruction is issued by one elected lane.
    uint32_t kv_cnt = 0;
    uint32_t q_use[NQ] = {0, 0}, p_use[NQ] = {0, 0}, o_use[NQ] = {0, 0};
    bool ok = true;
    // K-major SW128 descriptors of the Q tiles and of ring slot 0; a slot or a
    // 16-element K step only moves the start address (16-byte units).  Each
    // group of products is issued by one elected lane (one election per group:
    // an election per instruction measured 2.5 % slower on the whole kernel).
    const uint64_t dQ0 = sdesc(sQ, 16, 1024);
    const uint64_t dKV0 = sdesc(sKV, 16, 1024);
    const uint64_t dV0 = sdesc(sKV, BOX_BYTES, 1024);
    constexpr uint32_t TILE16 = C::TILE_BYTES >> 4;
    auto qk = [&](int t, uint32_t kslot) {
      const uint64_t a = dQ0 + (uint64_t)(t * TILE16);
      const uint64_t b = dKV0 + (uint64_t)(kslot * TILE16);
      const uint32_t d = tmem + t * BM;
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (uint32_t)((kk >> 2) * (BOX_BYTES >> 4) + (kk & 3) * 2);
          mma_ss(d, a + off, b + off, IDESC_QK, kk > 0 ? 1u : 0u);
        }
      }
      __syncwarp();
    };
    auto pv = [&](int t, uint32_t vslot, bool acc0) {
      const uint64_t b = dV0 + (uint64_t)(vslot * TILE16);
      const uint32_t d = tmem + 2 * BM + t * D, a = tmem + t * BM;
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          mma_ts(d, a + kk * 8, b + (uint64_t)(kk * 128), IDESC_PV, (acc0 || kk > 0) ? 1u : 0u);
      }
      __syncwarp();
    };
    uint32_t uq_pos = 0;
    while (ok) {
      const uint32_t qs = uq_pos % UQ_DEPTH;
      ok = wait_bar(bar(C::UQ_FULL + qs), (uq_pos / UQ_DEPTH) & 1u, abort_flag, limit);
      if (!ok) break;
      const int u = uq_ids[qs];
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::UQ_EMPTY + qs));
      ++uq_pos;
      if (u >= p.total_units) break;
      const Unit un = decode_unit<KIND>(p, u);
      const int n = max(un.n[0], un.n[1]);
      if (KIND == PACKED && n == 0) continue;   // an empty sequence of a variable-length batch
#pragma unroll
      for (int t = 0; t < NQ; ++t) {
        if (un.n[t] == 0 || !ok) continue;
        ok = wait_bar(bar(C::Q_FULL + t), q_use[t] & 1u, abort_flag, limit);
        ++q_use[t];
      }
      if (!ok) break;
      // S_t = Q_t K_0^T
      uint32_t kslot = kv_cnt % C::NSLOT;
      ok = wait_bar(bar(C::KV_FULL + kslot), (kv_cnt / C::NSLOT) & 1u, abort_flag, limit);
      if (!ok) break;
      ++kv_cnt;
      tc_fence_after();
#pragma unroll
      for (int t = 0; t < NQ; ++t) {
        if (un.n[t] == 0) continue;
        qk(t, kslot);
        tc_commit_elect(bar(C::S_FULL + t));
        // packed batch: Q_t is read by no later MMA, so the producer may load
        // the next unit's Q_t as soon as this one completes
        if (ROWSTORE && un.n[t] == 1) tc_commit_elect(bar(C::Q_EMPTY + t));
      }
      tc_commit_elect(bar(C::KV_EMPTY + kslot));
      for (int j = 0; j < n && ok; ++j) {
        const uint32_t vslot = kv_cnt % C::NSLOT;
        ok = wait_bar(bar(C::KV_FULL + vslot), (kv_cnt / C::NSLOT) & 1u, abort_flag, limit);
        if (!ok) break;
        ++kv_cnt;
        bool k_ready = false;
        kslot = kv_cnt % C::NSLOT;
#pragma unroll
        for (int t = 0; t < NQ; ++t) {
          if (j >= un.n[t] || !ok) continue;
          ok = wait_bar(bar(C::P_FULL + t), p_use[t] & 1u, abort_flag, limit);
          if (!ok) break;
          ++p_use[t];
          if (j == 0) {
            ok = wait_bar(bar(C::O_EMPTY + t), (o_use[t] & 1u) ^ 1u, abort_flag, limit);
            if (!ok) break;
            ++o_use[t];
          }
          tc_fence_after();
          // O_t += P_t V_j   (P_t in TMEM, 16 keys = 8 packed columns per step)
          pv(t, vslot, j > 0);
          if (j + 1 == un.n[t]) tc_commit_elect(bar(C::O_FULL + t));   // O_t final: the epilogue may read it
          if (j + 1 < un.n[t]) {
            if (!k_ready) {
              ok = wait_bar(bar(C::KV_FULL + kslot), (kv_cnt / C::NSLOT) & 1u, abort_flag, limit);
              if (!ok) break;
              ++kv_cnt;
              k_ready = true;
              tc_fence_after();
            }
            // S_t = Q_t K_{j+1}^T; its commit also covers PV_t(j), so the
            // softmax may rescale O_t once it has seen S_t(j+1).
            qk(t, kslot);
            tc_commit_elect(bar(C::S_FULL + t));
            if (ROWSTORE && j + 2 == un.n[t]) tc_commit_elect(bar(C::Q_EMPTY + t));   // last read of Q_t
          }
        }
        if (!ok) break;
        tc_commit_elect(bar(C::KV_EMPTY + vslot));
        if (k_ready) tc_commit_elect(bar(C::KV_EMPTY + kslot));
      }
    }
    // Drain: every MMA this warp issued has completed before TMEM is freed.
    tc_commit_elect(bar(C::DRAIN));
    if (lane == 0) drain_wait(bar(C::DRAIN), 0, limit);
    __syncwarp();
   }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REGS_SOFTMAX));
    // ------------------------------------------------------------------ softmax warpgroups
    const int t = warp >> 2;               // query tile of this warpgroup
    const int quad = warp & 3;             // TMEM lane quadrant
    const int rit = quad * 32 + lane;      // row inside the tile
    const uint32_t lane_bits = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tmem + lane_bits + t * BM;
    const uint32_t tO = tmem + lane_bits + 2 * BM + t * D;
    const float c = p.scale_log2;
    const float tau = p.rescale_log2, tau_pow2 = p.rescale_pow2;
    const float headroom = BF16 ? p.headroom_log2 : 0.f;
    uint32_t s_use = 0, o_use = 0, e_use = 0;
    bool ok = true;
    uint8_t* sQt = smem + C::SMEM_Q + t * C::TILE_BYTES;

    uint32_t uq_pos = 0;
    while (ok) {
      const uint32_t qs = uq_pos % UQ_DEPTH;
      ok = wait_bar(bar(C::UQ_FULL + qs), (uq_pos / UQ_DEPTH) & 1u, abort_flag, limit);
      if (!ok) break;
      const int u = uq_ids[qs];
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::UQ_EMPTY + qs));
      ++uq_pos;
      if (u >= p.total_units) break;
      const Unit un = decode_unit<KIND>(p, u);
      const int nt = t ? un.n[1] : un.n[0];
      if (nt == 0) continue;
      const int row = un.r0 + t * BM + rit;          // query row of this thread
      const int first_row = un.r0 + t * BM;
      // the rows the causal mask is taken at (a ring step's segment offsets them)
      const int mrow = KIND == RING ? row + un.coff : row;
      const int mfirst = KIND == RING ? first_row + un.coff : first_row;
      const bool causal = KIND == RING ? (un.causal != 0) : (p.causal != 0);
      float m = -INFINITY;                           // running max, log2 domain
      float l = 0.f;                                 // running exp-sum (for the LSE)
      float ln = 0.f;                                // l with each tile's top weight as rounded in P (for O)
      float m_use = 0.f;
      for (int j = 0; j < nt; ++j) {
        if constexpr (KIND == RING) {
          // the running O row the epilogue merges with: into L2 while the last tile is computed
          if (j + 1 == nt && p.split_n == 0 && !((un.seg ? p.seg_flags[1] : p.seg_flags[0]) & 1) && row < un.sq) {
            const float* a = p.acc + (size_t)un.b * p.o_bs + (size_t)un.h * p.o_hs + (size_t)(un.ob + row) * p.o_rs;
#pragma unroll
            for (int i = 0; i < D / 32; ++i) prefetch_l2(a + 32 * i);
          }
        }
        // S_t(j) is complete; its commit also covers P_t(j-1) V(j-1), so O_t is settled.
        ok = wait_bar(bar(C::S_FULL + t), s_use & 1u, abort_flag, limit);
        if (!ok) break;
        ++s_use;
        tc_fence_after();
        const int c0 = j * BN;
        const bool masked = (c0 + BN > un.sk) || (causal && (c0 + BN - 1 > mfirst));
        const float cc = masked ? 1.f : c;
        int lim = un.sk - 1 - c0;
        if (causal) lim = min(lim, mrow - c0);
        // this row of S_t from TMEM; diagonal / ragged tiles become scaled logits
        // with masked entries at -inf
        auto load_s = [&](uint32_t (&sr)[BN]) {
          tmem_ld_cols<BN / 32>(tS, sr);
          if (masked) {
#pragma unroll
            for (int k = 0; k < BN; ++k)
              sr[k] = __float_as_uint((k > lim) ? -INFINITY : __uint_as_float(sr[k]) * c);
          }
        };
        uint32_t sr[BN];
        uint32_t pk[BN / 2];
        load_s(sr);
        // P = 2^(s * cc - m), packed in registers; written to TMEM (the first
        // 64 columns of S_t) only once accepted.  From the second tile on, the
        // exponentials are taken against the current reference m straight
        // away: the reference must move only if this tile's max exceeds it by
        // more than tau, which shows as a weight above 2^tau.  Then (rarely)
        // the warp reloads S (still intact in
        // TMEM), takes the exact tile max, moves m and recomputes P.  The first
        // tile of a unit starts from the exact max.
        float p_top = 0.f, rowsum = 0.f;
        bool grow = false;
        const float m_prev = m;
        bool exact = (j == 0);
        if (!exact) {
          rowsum = exp_pack_row<BF16, EMU_PAIRS>(sr, cc, -m_use, pk, p_top);
          exact = __any_sync(0xffffffffu, !(p_top <= tau_pow2));
          if (exact) load_s(sr);
        }
        if (exact) {
          const float m_blk = row_max_scaled(sr, cc);
          const float m_cand = fmaxf(m, m_blk);
          grow = (m == -INFINITY) || (m_cand > m + tau) || !(p_top <= tau_pow2);
          // bf16 keeps the fp32 exponent range, so the new reference is set
          // above the max (weights <= 2^-headroom) and later tiles may grow by
          // headroom + tau before the next move; fp16 keeps the max.
          if (grow) m = m_cand + headroom;
          m_use = (m == -INFINITY) ? 0.f : m;
          rowsum = exp_pack_row<BF16, EMU_PAIRS>(sr, cc, -m_use, pk, p_top);
        }
#pragma unroll
        for (int h2 = 0; h2 < BN / 64; ++h2)
          tmem_st32(tS + h2 * 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32 * h2]));
        const float alpha = grow ? ex2(m_prev - m_use) : 1.f;   // 0 when m_prev = -inf
        // P enters P.V rounded to the input dtype.  The largest weight of the
        // tile can exceed 1 (stale max), where rounding is not exact; adding its
        // rounding error to the normaliser makes O divide by the same value it
        // multiplied by, so a dominant key carries no extra error.
        const float corr = round_to_input<BF16>(p_top) - p_top;
        l = l * alpha + rowsum;
        ln = ln * alpha + rowsum + corr;
        if (p.counts != nullptr && j > 0) {
          const bool any_grow = __any_sync(0xffffffffu, grow);
          const bool near = __any_sync(0xffffffffu, !exact && p_top > 0.5f * tau_pow2);
          if (lane == 0) {
            atomicAdd(&p.counts[0], 1ull);
            if (exact) atomicAdd(&p.counts[1], 1ull);
            if (any_grow) atomicAdd(&p.counts[2], 1ull);
            if (near) atomicAdd(&p.counts[3], 1ull);
          }
        }
        if (j > 0 && __any_sync(0xffffffffu, grow)) {
          uint32_t orow[D];
          tmem_ld_cols<D / 32>(tO, orow);
          const uint64_t a2 = f2pack(alpha, alpha);
#pragma unroll
          for (int i = 0; i < D / 2; ++i) {
            float o0, o1;
            f2unpack(fmul2(f2pack(__uint_as_float(orow[2 * i]), __uint_as_float(orow[2 * i + 1])), a2), o0, o1);
            orow[2 * i] = __float_as_uint(o0);
            orow[2 * i + 1] = __float_as_uint(o1);
          }
#pragma unroll
          for (int q4 = 0; q4 < D / 32; ++q4)
            tmem_st32(tO + q4 * 32, *reinterpret_cast<uint32_t(*)[32]>(&orow[32 * q4]));
        }
        tmem_wait_st();
        tc_fence_before();
        // every lane's P (and rescaled O) stores are complete: one arrival per warp
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(C::P_FULL + t));
      }
      if (!ok) break;

      // ---------------------------------------------------------------- epilogue
      ok = wait_bar(bar(C::O_FULL + t), o_use & 1u, abort_flag, limit);
      if (!ok) break;
      ++o_use;
      tc_fence_after();
      const bool store_row = row < un.sq;
      if constexpr (KIND == RING) {
        // Ring step: merged with the running result of the rows (LSE a, fp32
        // O in acc) unless this is their first result: the merged LSE is
        // log2(2^a + 2^lse2) and each part is weighted by 2^(its LSE - merged).
        // Stored as the running result (fp32) or, at the rows' last segment,
        // as the output in the input dtype; each thread stores its own row.
        // (a split-KV split is always its rows' first result and never their last)
        const int seg_flags = p.split_n > 0 ? 1 : (un.seg ? p.seg_flags[1] : p.seg_flags[0]);
        const bool final_o = (seg_flags & 2) != 0;
        const bool merge = !(seg_flags & 1) && store_row;
        const size_t lse_at = (size_t)un.b * p.lse_bs + (size_t)un.h * p.lse_hs + un.ob + row;
        const size_t e = (size_t)un.b * p.o_bs + (size_t)un.h * p.o_hs + (size_t)(un.ob + row) * p.o_rs;
        uint8_t* orow = p.o + e * 2;
        float* arow = p.acc + e;
        float lse2 = m_use + lg2(l);          // this segment's LSE (log2 units)
        float w_o = 1.f / ln, w_run = 0.f;    // O = w_o * O_tmem + w_run * running O
        if (merge) {
          const float a = p.lse[lse_at] * 1.44269504088896340736f;
          const float mx = fmaxf(a, lse2);
          const float ea = ex2(a - mx), eb = ex2(lse2 - mx);
          const float inv = 1.f / (ea + eb);
          w_run = ea * inv;
          w_o *= eb * inv;
          lse2 = mx + lg2(ea + eb);
        }
        uint32_t r[32];
        // (kept rolled: unrolled, the running O loads of every chunk are
        // hoisted together and the registers spill)
#pragma unroll 1
        for (int q4 = 0; q4 < D / 32; ++q4) {
          tmem_ld32(tO + q4 * 32, r);
          tmem_wait_ld();
          reg_fence(r);
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * w_o);
          if (merge) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const float4* src = reinterpret_cast<const float4*>(arow) + q4 * 8 + h * 4;
              float4 run[4];     // 16 columns of the running O row
#pragma unroll
              for (int i = 0; i < 4; ++i) run[i] = src[i];
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                uint32_t* x = &r[16 * h + 4 * i];
                x[0] = __float_as_uint(fmaf(run[i].x, w_run, __uint_as_float(x[0])));
                x[1] = __float_as_uint(fmaf(run[i].y, w_run, __uint_as_float(x[1])));
                x[2] = __float_as_uint(fmaf(run[i].z, w_run, __uint_as_float(x[2])));
                x[3] = __float_as_uint(fmaf(run[i].w, w_run, __uint_as_float(x[3])));
              }
            }
          }
          if (!store_row) continue;
          if (final_o) {
            uint32_t w[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) w[i] = pack2<BF16>(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
            uint4* dst = reinterpret_cast<uint4*>(orow + q4 * 64);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(arow) + q4 * 8;
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[i] = make_uint4(r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]);
          }
        }
        if (store_row) p.lse[lse_at] = lse2 * 0.69314718055994530942f;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(C::O_EMPTY + t));
      } else {
        const float inv_l = 1.f / ln;
        // Dense batch: O is staged (swizzled) in the Q tile's buffer and
        // stored by TMA; the buffer is released once the store has read it.
        // Packed (variable-length) batch: each thread stores its own row
        // from registers -- a tile may end inside the sequence, where a TMA
        // store would also write the next sequence's rows -- and the MMA warp
        // has already released the Q buffer after its last read.
        uint8_t* orow = nullptr;
        if constexpr (KIND == PACKED) orow = p.o + ((size_t)(un.rb + row) * p.H + un.h) * (D * 2);
        {
          uint32_t r[32];
#pragma unroll
          for (int q4 = 0; q4 < D / 32; ++q4) {
            tmem_ld32(tO + q4 * 32, r);
            tmem_wait_ld();
            reg_fence(r);
            uint32_t w[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              w[i] = pack2<BF16>(__uint_as_float(r[2 * i]) * inv_l, __uint_as_float(r[2 * i + 1]) * inv_l);
            if constexpr (KIND == PACKED) {
              if (store_row) {
                uint4* dst = reinterpret_cast<uint4*>(orow + q4 * 64);
#pragma unroll
                for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
              }
            } else {
              // row rit of box q4/2, 16-byte chunks (q4&1)*4 + i, 128-byte swizzle
              uint8_t* rowp = sQt + (q4 >> 1) * BOX_BYTES + rit * 128;
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int chunk = ((q4 & 1) * 4 + i) ^ (rit & 7);
                *reinterpret_cast<uint4*>(rowp + chunk * 16) =
                    make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(C::O_EMPTY + t));
        if constexpr (!ROWSTORE) {
          fence_proxy_async_smem();
          mbar_arrive(bar(C::EPI + t));
        }
        if (store_row) {
          const float lse = (m_use + lg2(l)) * 0.69314718055994530942f;
          p.lse[(size_t)un.b * p.lse_bs + (size_t)un.h * p.lse_hs + un.rb + row] = lse;
        }
      }
      if constexpr (!ROWSTORE) {
        if (rit == 0) {
          // one thread stores the tile once all 128 rows are staged
          drain_wait(bar(C::EPI + t), e_use & 1u, limit);
          for (int bx = 0; bx < C::NBOX; ++bx)
            tma_store_4d(&tmO, smem_u32(sQt + bx * BOX_BYTES), bx * 64, p.bhsd ? first_row : un.h,
                         p.bhsd ? un.h : first_row, un.tb);
          tma_store_commit();
          tma_store_wait_read();
          mbar_arrive(bar(C::Q_EMPTY + t));
        }
        ++e_use;
      }
      __syncwarp();
    }
    if constexpr (!ROWSTORE) {
      if (rit == 0) tma_store_wait_all();
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace fa

// ============================================================================= host side

namespace {

thread_local int t_last_cuda_error = 0;

fa_status cuda_fail(int err) {
  t_last_cuda_error = err;
  return FA_ERR_CUDA;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn(int* err) {
  static EncodeTiledFn fn = nullptr;
  static int init_err = 0;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !ptr) {
      init_err = (e != cudaSuccess) ? (int)e : 999;
      return;
    }
    fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  *err = init_err;
  return fn;
}

// A [B, S, H, D] (BSND) or [B, H, S, D] (BHSD) tensor seen as 4-D for TMA,
// dims in memory order, box_rows x 64-column boxes with a 128-byte swizzle.
fa_status make_map(CUtensorMap* map, const void* base, fa_dtype dt, fa_layout lay, int64_t B, int64_t H,
                   int64_t S, int64_t D, int box_rows = fa::BM) {
  int err = 0;
  EncodeTiledFn enc = get_encode_fn(&err);
  if (!enc) return cuda_fail(err);
  cuuint64_t dims[4], strides[3];
  cuuint32_t box[4];
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  if (lay == FA_BHSD) {
    dims[0] = D; dims[1] = S; dims[2] = H; dims[3] = B;
    strides[0] = D * 2; strides[1] = S * D * 2; strides[2] = H * S * D * 2;
    box[0] = 64; box[1] = (cuuint32_t)box_rows; box[2] = 1; box[3] = 1;
  } else {
    dims[0] = D; dims[1] = H; dims[2] = S; dims[3] = B;
    strides[0] = D * 2; strides[1] = H * D * 2; strides[2] = S * H * D * 2;
    box[0] = 64; box[1] = 1; box[2] = (cuuint32_t)box_rows; box[3] = 1;
  }
  const CUtensorMapDataType t =
      dt == FA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUresult r = enc(map, t, 4, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cuda_fail((int)r);
  return FA_OK;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

fa_status check_device_ptr(const void* ptr, int device) {
  cudaPointerAttributes attr;
  cudaError_t e = cudaPointerGetAttributes(&attr, ptr);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return cuda_fail((int)e);
  }
  if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged) return FA_ERR_NOT_DEVICE_POINTER;
  if (attr.device != device) return FA_ERR_NOT_DEVICE_POINTER;
  return FA_OK;
}

struct DeviceInfo {
  int sms = 0;
  bool configured[12] = {};   // per kernel instantiation: shared-memory attribute set
};

template <int D, bool BF16, int KIND>
fa_status launch(const fa::Params& prm, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                 const CUtensorMap& o, int grid, bool* configured, cudaStream_t stream) {
  auto kern = fa::fa_fwd_kernel<D, BF16, KIND>;
  const int smem = fa::Cfg<D>::SMEM_BYTES;
  if (!*configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail((int)e);
    *configured = true;
  }
  kern<<<grid, fa::NUM_THREADS, smem, stream>>>(prm, q, k, v, o);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail((int)e);
  return FA_OK;
}

constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

constexpr size_t kWorkspaceBytes = 16;  // the work counter of the dynamic schedule (4 bytes used)

// Validates the arguments, builds the tensor maps and launches the kernel.
// sched: the dynamic-schedule counter in device memory (zeroed here, on the
// stream, before the launch), or nullptr for the static schedule.
// The current device, its SM count, and every non-null pointer on it.
fa_status device_checks(const void* const* ptrs, int n, int* dev_out, int* sms_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail((int)e);
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  for (int i = 0; i < n; ++i) {
    if (!ptrs[i]) continue;   // optional arguments (the work counter) may be null
    fa_status st = check_device_ptr(ptrs[i], dev);
    if (st != FA_OK) return st;
  }
  std::lock_guard<std::mutex> g(g_dev_mu);
  if (g_dev[dev].sms == 0) {
    e = cudaDeviceGetAttribute(&g_dev[dev].sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail((int)e);
  }
  *dev_out = dev;
  *sms_out = g_dev[dev].sms;
  return FA_OK;
}

// Persistent grid of min(#SMs, #units) CTAs; zeroes the work counter first.
fa_status launch_units(fa::Params& prm, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                       const CUtensorMap& mo, int64_t D, fa_dtype dtype, unsigned int* sched, int dev, int sms,
                       void* stream) {
  const int grid = (int)(prm.total_units < sms ? prm.total_units : sms);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // With no more units than CTAs every CTA takes exactly its first unit, and
  // the work counter would only be read to find nothing left: the launch then
  // runs the static schedule (the same units, the same results) and the
  // counter is not zeroed, which saves a memset on small, latency-bound calls.
  if (prm.total_units <= grid) sched = nullptr;
  prm.sched = sched;
  if (sched) {
    cudaError_t e = cudaMemsetAsync(sched, 0, sizeof(unsigned int), s);
    if (e != cudaSuccess) return cuda_fail((int)e);
  }
  bool* cfg = g_dev[dev].configured;
  using fa::DENSE;
  using fa::PACKED;
  using fa::RING;
  if (prm.nseg > 0) {
    if (D == 128)
      return dtype == FA_BF16 ? launch<128, true, RING>(prm, mq, mk, mv, mo, grid, &cfg[8], s)
                              : launch<128, false, RING>(prm, mq, mk, mv, mo, grid, &cfg[9], s);
    return dtype == FA_BF16 ? launch<64, true, RING>(prm, mq, mk, mv, mo, grid, &cfg[10], s)
                            : launch<64, false, RING>(prm, mq, mk, mv, mo, grid, &cfg[11], s);
  }
  if (prm.cu_q) {
    if (D == 128)
      return dtype == FA_BF16 ? launch<128, true, PACKED>(prm, mq, mk, mv, mo, grid, &cfg[4], s)
                              : launch<128, false, PACKED>(prm, mq, mk, mv, mo, grid, &cfg[5], s);
    return dtype == FA_BF16 ? launch<64, true, PACKED>(prm, mq, mk, mv, mo, grid, &cfg[6], s)
                            : launch<64, false, PACKED>(prm, mq, mk, mv, mo, grid, &cfg[7], s);
  }
  if (D == 128)
    return dtype == FA_BF16 ? launch<128, true, DENSE>(prm, mq, mk, mv, mo, grid, &cfg[0], s)
                            : launch<128, false, DENSE>(prm, mq, mk, mv, mo, grid, &cfg[1], s);
  return dtype == FA_BF16 ? launch<64, true, DENSE>(prm, mq, mk, mv, mo, grid, &cfg[2], s)
                          : launch<64, false, DENSE>(prm, mq, mk, mv, mo, grid, &cfg[3], s);
}

// Heads whose K and V (Sk keys each) fit together in about 48 MB of L2.
int l2_group_heads(int64_t Sk, int64_t D, int64_t BH) {
  const int64_t kv_head_bytes = 2 * Sk * D * 2;
  int64_t gh = ((int64_t)48 << 20) / (kv_head_bytes > 0 ? kv_head_bytes : 1);
  if (gh < 1) gh = 1;
  if (gh > BH) gh = BH;
  return (int)gh;
}

// Self-test settings: a kernel that withholds its loads, with a short wait limit.
struct SelfTest {
  unsigned long long wait_limit_ns;
};

// The lazy rescale's settings and the optional branch statistics (fa_fwd_options).
struct SoftmaxOpts {
  float rescale_log2 = fa::RESCALE_LOG2_DEFAULT;
  float headroom_log2 = fa::HEADROOM_LOG2_DEFAULT;
  unsigned long long* counts = nullptr;
};

void set_softmax_params(fa::Params& prm, const SoftmaxOpts& so) {
  prm.rescale_log2 = so.rescale_log2;
  prm.rescale_pow2 = exp2f(so.rescale_log2);
  prm.headroom_log2 = so.headroom_log2;
  prm.counts = so.counts;
}

// Every check of a dense forward call's arguments that needs no device, in
// the order fa_fwd applies them.  FA_OK with *noop set: the call has no query
// rows and nothing to do (the pointers are then not looked at).
fa_status host_checks(const void* q, const void* k, const void* v, const void* o, const float* lse, int64_t B,
                      int64_t H, int64_t Sq, int64_t Sk, int64_t D, fa_layout layout, float scale, fa_dtype dtype,
                      bool* noop) {
  *noop = false;
  if (B <= 0 || H <= 0 || Sq < 0 || Sk <= 0 || D <= 0) return FA_ERR_INVALID_ARG;
  if (layout != FA_BSND && layout != FA_BHSD) return FA_ERR_INVALID_ARG;
  if (dtype != FA_FP16 && dtype != FA_BF16) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  // TMA coordinates and the schedule use 32-bit integers
  const int64_t lim = (int64_t)1 << 30;
  if (B >= lim || H >= lim || Sq >= lim || Sk >= lim || B * H >= lim) return FA_ERR_UNSUPPORTED;
  const int64_t nqb = (Sq + fa::UNIT_ROWS - 1) / fa::UNIT_ROWS;
  if (B * H * nqb >= lim) return FA_ERR_UNSUPPORTED;
  if (Sq == 0) {
    *noop = true;
    return FA_OK;
  }
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v) |
       reinterpret_cast<uintptr_t>(o)) & 15u)
    return FA_ERR_MISALIGNED;
  if (reinterpret_cast<uintptr_t>(lse) & 3u) return FA_ERR_MISALIGNED;
  const size_t qbytes = (size_t)(B * H * Sq * D) * 2, kvbytes = (size_t)(B * H * Sk * D) * 2;
  const size_t lbytes = (size_t)(B * H * Sq) * 4;
  if (overlaps(o, qbytes, q, qbytes) || overlaps(o, qbytes, k, kvbytes) || overlaps(o, qbytes, v, kvbytes) ||
      overlaps(lse, lbytes, q, qbytes) || overlaps(lse, lbytes, k, kvbytes) ||
      overlaps(lse, lbytes, v, kvbytes) || overlaps(lse, lbytes, o, qbytes))
    return FA_ERR_ALIAS;
  return FA_OK;
}

// head_begin / head_count: the flattened heads b * H + h the launch computes
// (all of them: 0 / -1); the tensors are the whole [B, H] problem either way.
fa_status fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t H,
                   int64_t Sq, int64_t Sk, int64_t D, fa_layout layout, int causal, float scale, fa_dtype dtype,
                   unsigned int* sched, void* stream, const SelfTest* selftest = nullptr, int64_t head_begin = 0,
                   int64_t head_count = -1, const SoftmaxOpts& so = SoftmaxOpts()) {
  // ---- arguments that need no device
  bool noop = false;
  fa_status hst = host_checks(q, k, v, o, lse, B, H, Sq, Sk, D, layout, scale, dtype, &noop);
  if (hst != FA_OK || noop) return hst;
  const int64_t nqb = (Sq + fa::UNIT_ROWS - 1) / fa::UNIT_ROWS;
  if (head_count < 0) head_count = B * H;
  if (head_begin < 0 || head_begin > B * H || head_count > B * H - head_begin) return FA_ERR_INVALID_ARG;
  if (head_count == 0) return FA_OK;

  // ---- device checks
  int dev = 0, sms = 0;
  const void* ptrs[7] = {q, k, v, o, lse, sched, so.counts};
  fa_status st = device_checks(ptrs, 7, &dev, &sms);
  if (st != FA_OK) return st;

  CUtensorMap mq, mk, mv, mo;
  if ((st = make_map(&mq, q, dtype, layout, B, H, Sq, D)) != FA_OK) return st;
  if ((st = make_map(&mk, k, dtype, layout, B, H, Sk, D)) != FA_OK) return st;
  if ((st = make_map(&mv, v, dtype, layout, B, H, Sk, D)) != FA_OK) return st;
  if ((st = make_map(&mo, o, dtype, layout, B, H, Sq, D)) != FA_OK) return st;

  fa::Params prm{};   // no ring segments
  prm.lse = lse;
  prm.cu_q = nullptr;
  prm.cu_k = nullptr;
  prm.total_q = 0;
  prm.total_k = 0;
  prm.o = static_cast<uint8_t*>(o);
  prm.lse_bs = H * Sq;
  prm.lse_hs = Sq;
  prm.B = (int)B;
  prm.H = (int)H;
  prm.Sq = (int)Sq;
  prm.Sk = (int)Sk;
  prm.nqb = (int)nqb;
  prm.tk = (int)((Sk + fa::BN - 1) / fa::BN);
  prm.bh = (int)head_count;
  prm.head0 = (int)head_begin;
  prm.group_heads = l2_group_heads(Sk, D, head_count);
  prm.total_units = (int)(head_count * nqb);
  prm.causal = causal ? 1 : 0;
  prm.bhsd = layout == FA_BHSD ? 1 : 0;
  prm.scale_log2 = (float)((double)scale * 1.4426950408889634074);
  prm.wait_limit_ns = 1000000000ull;  // one second; a normal wait lasts microseconds
  prm.withhold_loads = 0;
  set_softmax_params(prm, so);
  if (selftest) {
    prm.wait_limit_ns = selftest->wait_limit_ns;
    prm.withhold_loads = 1;
  }

  return launch_units(prm, mq, mk, mv, mo, D, dtype, sched, dev, sms, stream);
}

// ---------------------------------------------------------------------------
// Entry point without allocation (fa_fwd_noalloc).
//
// Some callers cannot give this library device memory: a plugin whose host
// framework owns every device allocation and hands over only the input and
// output buffers, or a real-time path that must not call the CUDA allocator
// (cudaMalloc can synchronise the device and fragment a fixed memory budget).
// For them the dynamic schedule's scratch -- its work counter -- lives in the
// fixed array below, which every GPU that loads this library holds until the
// process exits.  In host code the array's name is only a host-side stand-in;
// its device address comes from cudaGetSymbolAddress, once per device, with
// that device current, on the first fa_fwd_noalloc call there.
constexpr size_t kNoAllocScratchBytes = 256;   // capacity of the fixed scratch
// The schedule needs kWorkspaceBytes whatever the call's sizes, so the fixed
// array always suffices; a scratch need that grew with the sizes would have
// to be refused at run time instead.
static_assert(kWorkspaceBytes <= kNoAllocScratchBytes, "the fixed scratch cannot hold the schedule's counter");

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices];   // a device's looked-up address; null until a lookup succeeds

}  // namespace

static __device__ __align__(256) unsigned char fa_noalloc_scratch[kNoAllocScratchBytes];

namespace {

// Device address of fa_noalloc_scratch on `dev` (the current device).  Only a
// successful lookup is kept, so a failed one (say, attempted during a stream
// capture) is simply tried again by the next call.  `refresh` forces a new
// lookup: after cudaDeviceReset the module is loaded anew and a kept address
// may be stale.  nullptr with *err set on failure.
void* noalloc_scratch_address(int dev, bool refresh, int* err) {
  std::lock_guard<std::mutex> g(g_noalloc_mu);
  if (!g_noalloc_ptr[dev] || refresh) {
    void* ptr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&ptr, fa_noalloc_scratch);
    if (e != cudaSuccess) {
      cudaGetLastError();
      g_noalloc_ptr[dev] = nullptr;
      *err = (int)e;
      return nullptr;
    }
    g_noalloc_ptr[dev] = ptr;
  }
  return g_noalloc_ptr[dev];
}

}  // namespace

extern "C" {

fa_status fa_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B,
                         int64_t H, int64_t Sq, int64_t Sk, int64_t D, fa_layout layout, int causal, float scale,
                         fa_dtype dtype, void* stream) {
  // arguments that need no device, answered exactly as fa_fwd answers them
  bool noop = false;
  fa_status st = host_checks(q, k, v, o, lse, B, H, Sq, Sk, D, layout, scale, dtype, &noop);
  if (st != FA_OK || noop) return st;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail((int)e);
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  int err = 0;
  void* scratch = noalloc_scratch_address(dev, false, &err);
  if (!scratch) return cuda_fail(err);
  if (check_device_ptr(scratch, dev) != FA_OK) {
    // a kept address that no longer names device memory here: look it up once more
    scratch = noalloc_scratch_address(dev, true, &err);
    if (!scratch) return cuda_fail(err);
  }
  return fwd_impl(q, k, v, o, lse, B, H, Sq, Sk, D, layout, causal, scale, dtype,
                  static_cast<unsigned int*>(scratch), stream);
}

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t H,
                 int64_t Sq, int64_t Sk, int64_t D, fa_layout layout, int causal, float scale, fa_dtype dtype,
                 void* stream) {
  return fwd_impl(q, k, v, o, lse, B, H, Sq, Sk, D, layout, causal, scale, dtype, nullptr, stream);
}

fa_status fa_fwd_ws(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t H,
                    int64_t Sq, int64_t Sk, int64_t D, fa_layout layout, int causal, float scale, fa_dtype dtype,
                    void* workspace, size_t workspace_bytes, void* stream) {
  if (!workspace) {
    // the sizes may still make the call a no-op; otherwise a workspace is required
    if (Sq == 0 && B > 0 && H > 0 && Sk > 0) return FA_OK;
    return FA_ERR_INVALID_ARG;
  }
  if (workspace_bytes < kWorkspaceBytes) return FA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(workspace) & 15u) return FA_ERR_MISALIGNED;
  if (B > 0 && H > 0 && D > 0 && Sq > 0 && Sk > 0) {
    const size_t qbytes = (size_t)(B * H * Sq * D) * 2, kvbytes = (size_t)(B * H * Sk * D) * 2;
    const size_t lbytes = (size_t)(B * H * Sq) * 4;
    if ((q && overlaps(workspace, workspace_bytes, q, qbytes)) || (k && overlaps(workspace, workspace_bytes, k, kvbytes)) ||
        (v && overlaps(workspace, workspace_bytes, v, kvbytes)) || (o && overlaps(workspace, workspace_bytes, o, qbytes)) ||
        (lse && overlaps(workspace, workspace_bytes, lse, lbytes)))
      return FA_ERR_ALIAS;
  }
  return fwd_impl(q, k, v, o, lse, B, H, Sq, Sk, D, layout, causal, scale, dtype,
                  static_cast<unsigned int*>(workspace), stream);
}

size_t fa_fwd_workspace_size(void) { return kWorkspaceBytes; }

void fa_fwd_default_options(fa_fwd_options* opts) {
  if (!opts) return;
  opts->rescale_threshold_log2 = fa::RESCALE_LOG2_DEFAULT;
  opts->bf16_headroom_log2 = fa::HEADROOM_LOG2_DEFAULT;
  opts->branch_counts = nullptr;
}

fa_status fa_fwd_opts(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t H,
                      int64_t Sq, int64_t Sk, int64_t D, fa_layout layout, int causal, float scale, fa_dtype dtype,
                      const fa_fwd_options* opts, void* workspace, size_t workspace_bytes, void* stream) {
  SoftmaxOpts so;
  if (opts) {
    const float t = opts->rescale_threshold_log2, h = opts->bf16_headroom_log2;
    // weights against a stale reference reach 2^t, which must stay finite in fp16
    if (!(t >= 0.f && t <= 15.f) || !(h >= 0.f && h <= 16.f)) return FA_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(opts->branch_counts) & 7u) return FA_ERR_MISALIGNED;
    so.rescale_log2 = t;
    so.headroom_log2 = h;
    so.counts = opts->branch_counts;
  }
  unsigned int* sched = nullptr;
  if (workspace) {
    if (workspace_bytes < kWorkspaceBytes) return FA_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(workspace) & 15u) return FA_ERR_MISALIGNED;
    sched = static_cast<unsigned int*>(workspace);
  }
  if (B > 0 && H > 0 && D > 0 && Sq > 0 && Sk > 0) {
    const size_t qbytes = (size_t)(B * H * Sq * D) * 2, kvbytes = (size_t)(B * H * Sk * D) * 2;
    const size_t lbytes = (size_t)(B * H * Sq) * 4;
    const void* extra[2] = {workspace, so.counts};
    const size_t extra_bytes[2] = {workspace_bytes, 4 * sizeof(unsigned long long)};
    for (int i = 0; i < 2; ++i) {
      const void* x = extra[i];
      const size_t n = extra_bytes[i];
      if (x && ((q && overlaps(x, n, q, qbytes)) || (k && overlaps(x, n, k, kvbytes)) ||
                (v && overlaps(x, n, v, kvbytes)) || (o && overlaps(x, n, o, qbytes)) ||
                (lse && overlaps(x, n, lse, lbytes))))
        return FA_ERR_ALIAS;
    }
    if (workspace && so.counts && overlaps(workspace, workspace_bytes, so.counts, extra_bytes[1]))
      return FA_ERR_ALIAS;
  }
  return fwd_impl(q, k, v, o, lse, B, H, Sq, Sk, D, layout, causal, scale, dtype, sched, stream, nullptr, 0, -1,
                  so);
}

fa_status fa_fwd_heads(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t H,
                       int64_t Sq, int64_t Sk, int64_t D, fa_layout layout, int causal, float scale, fa_dtype dtype,
                       int64_t head_begin, int64_t head_count, void* workspace, size_t workspace_bytes,
                       void* stream) {
  if (head_begin < 0 || head_count < 0) return FA_ERR_INVALID_ARG;
  if (B > 0 && H > 0 && (head_begin > B * H || head_count > B * H - head_begin)) return FA_ERR_INVALID_ARG;
  if (!workspace)
    return fwd_impl(q, k, v, o, lse, B, H, Sq, Sk, D, layout, causal, scale, dtype, nullptr, stream, nullptr,
                    head_begin, head_count);
  if (workspace_bytes < kWorkspaceBytes) return FA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(workspace) & 15u) return FA_ERR_MISALIGNED;
  if (B > 0 && H > 0 && D > 0 && Sq > 0 && Sk > 0) {
    const size_t qbytes = (size_t)(B * H * Sq * D) * 2, kvbytes = (size_t)(B * H * Sk * D) * 2;
    const size_t lbytes = (size_t)(B * H * Sq) * 4;
    if ((q && overlaps(workspace, workspace_bytes, q, qbytes)) || (k && overlaps(workspace, workspace_bytes, k, kvbytes)) ||
        (v && overlaps(workspace, workspace_bytes, v, kvbytes)) || (o && overlaps(workspace, workspace_bytes, o, qbytes)) ||
        (lse && overlaps(workspace, workspace_bytes, lse, lbytes)))
      return FA_ERR_ALIAS;
  }
  return fwd_impl(q, k, v, o, lse, B, H, Sq, Sk, D, layout, causal, scale, dtype,
                  static_cast<unsigned int*>(workspace), stream, nullptr, head_begin, head_count);
}

fa_status fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse, const int32_t* cu_seqlens_q,
                        const int32_t* cu_seqlens_k, int64_t B, int64_t H, int64_t total_q, int64_t total_k,
                        int64_t max_seqlen_q, int64_t max_seqlen_k, int64_t D, int causal, float scale,
                        fa_dtype dtype, void* workspace, size_t workspace_bytes, void* stream) {
  // ---- arguments that need no device
  if (B <= 0 || H <= 0 || D <= 0 || total_q < 0 || total_k < 0 || max_seqlen_q < 0 || max_seqlen_k < 0)
    return FA_ERR_INVALID_ARG;
  if (dtype != FA_FP16 && dtype != FA_BF16) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  const int64_t lim = (int64_t)1 << 30;
  if (B >= lim || H >= lim || total_q >= lim || total_k >= lim || B * H >= lim) return FA_ERR_UNSUPPORTED;
  if (max_seqlen_q > total_q || max_seqlen_k > total_k) return FA_ERR_INVALID_ARG;
  const int64_t nqb = (max_seqlen_q + fa::UNIT_ROWS - 1) / fa::UNIT_ROWS;
  if (B * H * nqb >= lim) return FA_ERR_UNSUPPORTED;
  if (total_q == 0 || max_seqlen_q == 0) return FA_OK;   // no query rows
  if (max_seqlen_k == 0) return FA_ERR_INVALID_ARG;      // queries without keys
  if (!q || !k || !v || !o || !lse || !cu_seqlens_q || !cu_seqlens_k) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v) |
       reinterpret_cast<uintptr_t>(o)) & 15u)
    return FA_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(lse) | reinterpret_cast<uintptr_t>(cu_seqlens_q) |
       reinterpret_cast<uintptr_t>(cu_seqlens_k)) & 3u)
    return FA_ERR_MISALIGNED;
  if (workspace) {
    if (workspace_bytes < kWorkspaceBytes) return FA_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(workspace) & 15u) return FA_ERR_MISALIGNED;
  }
  const size_t qbytes = (size_t)(total_q * H * D) * 2, kvbytes = (size_t)(total_k * H * D) * 2;
  const size_t lbytes = (size_t)(total_q * H) * 4, cbytes = (size_t)(B + 1) * 4;
  const void* outs[2] = {o, lse};
  const size_t out_bytes[2] = {qbytes, lbytes};
  const void* ins[6] = {q, k, v, cu_seqlens_q, cu_seqlens_k, workspace};
  const size_t in_bytes[6] = {qbytes, kvbytes, kvbytes, cbytes, cbytes, workspace_bytes};
  for (int i = 0; i < 2; ++i)
    for (int j = 0; j < 6; ++j)
      if (ins[j] && overlaps(outs[i], out_bytes[i], ins[j], in_bytes[j])) return FA_ERR_ALIAS;
  if (overlaps(o, qbytes, lse, lbytes)) return FA_ERR_ALIAS;
  if (workspace)
    for (int j = 0; j < 5; ++j)
      if (overlaps(workspace, workspace_bytes, ins[j], in_bytes[j])) return FA_ERR_ALIAS;

  // ---- device checks
  int dev = 0, sms = 0;
  const void* ptrs[8] = {q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, workspace};
  fa_status st = device_checks(ptrs, 8, &dev, &sms);
  if (st != FA_OK) return st;

  // packed rows [total, H, D] are the BSND layout with one batch entry
  CUtensorMap mq, mk, mv, mo;
  if ((st = make_map(&mq, q, dtype, FA_BSND, 1, H, total_q, D)) != FA_OK) return st;
  if ((st = make_map(&mk, k, dtype, FA_BSND, 1, H, total_k, D)) != FA_OK) return st;
  if ((st = make_map(&mv, v, dtype, FA_BSND, 1, H, total_k, D)) != FA_OK) return st;
  if ((st = make_map(&mo, o, dtype, FA_BSND, 1, H, total_q, D)) != FA_OK) return st;

  fa::Params prm{};   // no ring segments
  prm.lse = lse;
  prm.cu_q = cu_seqlens_q;
  prm.cu_k = cu_seqlens_k;
  prm.total_q = (int)total_q;
  prm.total_k = (int)total_k;
  prm.o = static_cast<uint8_t*>(o);
  prm.o_bs = 0;                 // row r of head h at (r * H + h) * D
  prm.o_hs = D;
  prm.o_rs = H * D;
  prm.lse_bs = 0;
  prm.lse_hs = total_q;
  prm.B = (int)B;
  prm.H = (int)H;
  prm.Sq = (int)max_seqlen_q;
  prm.Sk = (int)max_seqlen_k;
  prm.nqb = (int)nqb;
  prm.tk = (int)((max_seqlen_k + fa::BN - 1) / fa::BN);
  prm.bh = (int)(B * H);
  prm.head0 = 0;
  prm.group_heads = l2_group_heads(max_seqlen_k, D, B * H);
  prm.total_units = (int)(B * H * nqb);
  prm.causal = causal ? 1 : 0;
  prm.bhsd = 0;
  prm.scale_log2 = (float)((double)scale * 1.4426950408889634074);
  prm.wait_limit_ns = 1000000000ull;
  prm.withhold_loads = 0;
  set_softmax_params(prm, SoftmaxOpts());
  return launch_units(prm, mq, mk, mv, mo, D, dtype, static_cast<unsigned int*>(workspace), dev, sms, stream);
}

fa_status fa_fwd_ring_step(const void* q, const void* k, const void* v, void* o, float* acc, float* lse, int64_t B,
                            int64_t H, int64_t Sq, int64_t Sk, int64_t D, int64_t rows, const fa_ring_segment* segs,
                            int nseg, fa_layout layout, float scale, fa_dtype dtype, void* workspace,
                            size_t workspace_bytes, void* stream) {
  bool noop = false;
  fa_status hst = host_checks(q, k, v, o, lse, B, H, Sq, Sk, D, layout, scale, dtype, &noop);
  if (hst != FA_OK) return hst;
  if (!segs || nseg < 1 || nseg > 2 || rows < 0 || rows > Sq) return FA_ERR_INVALID_ARG;
  if (noop || rows == 0) return FA_OK;
  bool need_acc = false;
  for (int s = 0; s < nseg; ++s) {
    const fa_ring_segment& g = segs[s];
    if (g.row0 < 0 || g.row0 > Sq - rows || g.key0 < 0 || g.keys < 1 || g.key0 > Sk - g.keys) return FA_ERR_INVALID_ARG;
    if ((g.first != 0 && g.first != 1) || (g.last != 0 && g.last != 1)) return FA_ERR_INVALID_ARG;
    if (g.causal_offset >= ((int64_t)1 << 30)) return FA_ERR_UNSUPPORTED;
    if (!g.first || !g.last) need_acc = true;
  }
  if (nseg == 2 && segs[0].row0 < segs[1].row0 + rows && segs[1].row0 < segs[0].row0 + rows)
    return FA_ERR_INVALID_ARG;   // two segments would write the same rows
  if (!workspace || workspace_bytes < kWorkspaceBytes) return FA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(workspace) & 15u) return FA_ERR_MISALIGNED;
  if (need_acc && !acc) return FA_ERR_INVALID_ARG;
  if (acc && (reinterpret_cast<uintptr_t>(acc) & 15u)) return FA_ERR_MISALIGNED;
  const size_t qbytes = (size_t)(B * H * Sq * D) * 2, kvbytes = (size_t)(B * H * Sk * D) * 2;
  const size_t lbytes = (size_t)(B * H * Sq) * 4, abytes = (size_t)(B * H * Sq * D) * 4;
  {
    const void* bufs[7] = {q, k, v, o, lse, acc, workspace};
    const size_t sizes[7] = {qbytes, kvbytes, kvbytes, qbytes, lbytes, abytes, workspace_bytes};
    for (int i = 5; i < 7; ++i)   // acc and the workspace against every other buffer
      for (int j = 0; j < 7; ++j)
        if (i != j && bufs[i] && bufs[j] && overlaps(bufs[i], sizes[i], bufs[j], sizes[j])) return FA_ERR_ALIAS;
  }

  int dev = 0, sms = 0;
  const void* ptrs[7] = {q, k, v, o, lse, acc, workspace};
  fa_status st = device_checks(ptrs, 7, &dev, &sms);
  if (st != FA_OK) return st;
  CUtensorMap mq, mk, mv, mo;
  if ((st = make_map(&mq, q, dtype, layout, B, H, Sq, D)) != FA_OK) return st;
  if ((st = make_map(&mk, k, dtype, layout, B, H, Sk, D)) != FA_OK) return st;
  if ((st = make_map(&mv, v, dtype, layout, B, H, Sk, D)) != FA_OK) return st;
  if ((st = make_map(&mo, o, dtype, layout, B, H, Sq, D)) != FA_OK) return st;

  // the segment with more keys first: its units are the longer ones
  int order[2] = {0, 1};
  if (nseg == 2 && segs[1].keys > segs[0].keys) {
    order[0] = 1;
    order[1] = 0;
  }
  int64_t max_keys = 0;
  for (int s = 0; s < nseg; ++s) max_keys = segs[s].keys > max_keys ? segs[s].keys : max_keys;
  const int64_t nqb = (rows + fa::UNIT_ROWS - 1) / fa::UNIT_ROWS;
  if (nseg * B * H * nqb >= ((int64_t)1 << 30)) return FA_ERR_UNSUPPORTED;

  fa::Params prm{};
  prm.lse = lse;
  prm.o = static_cast<uint8_t*>(o);
  if (layout == FA_BHSD) {
    prm.o_bs = H * Sq * D;
    prm.o_hs = Sq * D;
    prm.o_rs = D;
  } else {
    prm.o_bs = Sq * H * D;
    prm.o_hs = D;
    prm.o_rs = H * D;
  }
  prm.lse_bs = H * Sq;
  prm.lse_hs = Sq;
  prm.B = (int)B;
  prm.H = (int)H;
  prm.Sq = (int)rows;
  prm.Sk = (int)max_keys;
  prm.nqb = (int)nqb;
  prm.tk = (int)((max_keys + fa::BN - 1) / fa::BN);
  prm.bh = (int)(B * H);
  prm.head0 = 0;
  prm.group_heads = l2_group_heads(max_keys, D, B * H);
  prm.total_units = (int)(nseg * B * H * nqb);
  prm.causal = 0;
  prm.bhsd = layout == FA_BHSD ? 1 : 0;
  prm.scale_log2 = (float)((double)scale * 1.4426950408889634074);
  prm.wait_limit_ns = 1000000000ull;
  prm.withhold_loads = 0;
  set_softmax_params(prm, SoftmaxOpts());
  prm.nseg = nseg;
  prm.seg_units0 = (int)(B * H * nqb);
  for (int i = 0; i < nseg; ++i) {
    const fa_ring_segment& g = segs[order[i]];
    prm.seg_row0[i] = (int)g.row0;
    prm.seg_key0[i] = (int)g.key0;
    prm.seg_sk[i] = (int)g.keys;
    prm.seg_causal[i] = g.causal_offset >= 0 ? 1 : 0;
    prm.seg_coff[i] = g.causal_offset >= 0 ? (int)g.causal_offset : 0;
    prm.seg_flags[i] = (g.first ? 1 : 0) | (g.last ? 2 : 0);
  }
  prm.acc = acc;
  return launch_units(prm, mq, mk, mv, mo, D, dtype, static_cast<unsigned int*>(workspace), dev, sms, stream);
}

fa_status fa_selftest_wait_timeout(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B,
                                   int64_t H, int64_t Sq, int64_t Sk, int64_t D, fa_layout layout, int causal,
                                   float scale, fa_dtype dtype, uint32_t wait_limit_us, void* stream) {
  if (wait_limit_us < 1000u || wait_limit_us > 1000000u) return FA_ERR_INVALID_ARG;
  const SelfTest st{(unsigned long long)wait_limit_us * 1000ull};
  return fwd_impl(q, k, v, o, lse, B, H, Sq, Sk, D, layout, causal, scale, dtype, nullptr, stream, &st);
}

fa_status fa_device_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail((int)e);
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, fa::g_dev_error, sizeof(int));
  if (e != cudaSuccess) return cuda_fail((int)e);
  if (v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(fa::g_dev_error, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_fail((int)e);
    return (v & 1) ? FA_ERR_TIMEOUT : FA_ERR_INVALID_ARG;
  }
  return FA_OK;
}


fa_status fa_query_support(int64_t D, fa_dtype dtype) {
  if (dtype != FA_FP16 && dtype != FA_BF16) return FA_ERR_UNSUPPORTED;
  return (D == 64 || D == 128) ? FA_OK : FA_ERR_UNSUPPORTED;
}

const char* fa_status_string(fa_status status) {
  switch (status) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_NOT_DEVICE_POINTER: return "FA_ERR_NOT_DEVICE_POINTER";
    case FA_ERR_MISALIGNED: return "FA_ERR_MISALIGNED";
    case FA_ERR_ALIAS: return "FA_ERR_ALIAS";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT";
  }
  return "FA_ERR_UNKNOWN";
}

int fa_last_cuda_error(void) { return t_last_cuda_error; }

int fa_version(void) { return FA_VERSION; }

}  // extern "C"

// The backward pass (gradients) shares this translation unit's helpers.
#include "fa_bwd_impl.cuh"
#include "fa_merge_impl.cuh"
#include "fa_proj_impl.cuh"
