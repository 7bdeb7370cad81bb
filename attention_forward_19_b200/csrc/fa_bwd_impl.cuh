// fa_bwd_impl.cuh -- backward pass of the attention forward (dQ, dK, dV) for
// sm_100a and its C ABI.  Included at the end of fa_fwd.cu: one translation
// unit, sharing the PTX helpers, the tensor-map encoder, the host checks and
// the device error word.
//
// What is computed (the chain rule through O = softmax(S) V, S = scale Q K^T
// with the causal mask), with the weights recomputed from Q, K and the
// forward's log-sum-exp instead of stored (page "FlashAttention in
// ops-transformer on Ascend NPU" (ai6s.net/6a0d3bfb), section "how FA runs on
// the NPU": recomputation in the backward):
//   P = exp(S - LSE),  D_i = sum_d dO_id O_id,  dP = dO V^T,
//   dS = P * (dP - D),  dV = P^T dO,  dK = scale dS^T Q,  dQ = scale dS K.
//
// Design: deterministic, no atomics (page "catlass FlashAttention template
// tuning" (hwcomputing.csdn.net/6a0d4681), section on the backward: a
// `deterministic` switch between atomic adds and ordered accumulation).
//   1. prep kernel: D_i and LSE_i * log2(e), per row, into the workspace
//      (each head padded to whole 128-row tiles, padding +inf / 0).
//   2. dK/dV kernel, one CTA per 128-key tile: S^T = K Q_i^T and
//      dP^T = V dO_i^T for every visible query tile i put the keys on the TMEM
//      lanes; two threads per key (one per half of the query columns) compute
//      P^T and dS^T, write them (16-bit) over the S^T / dP^T columns they read
//      themselves, and dV += P^T dO_i,
//      dK += dS^T Q_i take them as the TMEM operand -- the same MMA forms as
//      the forward's O += P V.
//   3. dQ kernel, one CTA per 128-query tile: S = Q K_j^T, dP = dO V_j^T,
//      two threads per query row compute dS, and dQ += dS K_j.
// S and dP are computed by both kernels (7 tile products instead of 5): the
// price of having every gradient row owned by exactly one CTA.

namespace fa {
namespace bwd {

// Warps 0-7: two compute warpgroups on the same tile (warps w and w + 4 read
// the same TMEM lanes, one row each; group g takes columns [64 g, 64 g + 64)).
// Warp 8: loads.  Warp 9: MMA.
constexpr int THREADS = 320;
constexpr int LOAD_WARP = 8;
constexpr int MMA_WARP = 9;
constexpr int NSTAGE = 2;      // streamed tile pairs in flight
// The MMA warp issues step n + 1's first products before step n's last ones
// (which release step n's stage), so two stages are the minimum.
static_assert(NSTAGE >= 2, "the overlapped issue order needs two streamed stages");

template <int D>
struct Cfg {
  static constexpr int TILE = BM * D * 2;      // one 128-row tile
  static constexpr int NBOX = D / 64;
  static constexpr int IN_FULL = 0;            // the CTA's two fixed tiles
  static constexpr int ST_FULL = 1;            // a streamed stage (two tiles, + two vectors for dK/dV)
  static constexpr int ST_EMPTY = ST_FULL + NSTAGE;
  static constexpr int S_FULL = ST_EMPTY + NSTAGE;   // S^T (dK/dV) or S and dP (dQ) of a step are in TMEM
  static constexpr int DP_FULL = S_FULL + 1;         // dP^T of a step is in TMEM (dK/dV)
  static constexpr int RD_A = DP_FULL + 1;           // dQ: both groups have read S and dP (256 arrivals)
  static constexpr int W_A = RD_A + 1;               // P^T (dK/dV) or dS (dQ) written: 256
  static constexpr int W_B = W_A + 1;                // dS^T written (dK/dV): 256
  static constexpr int ACC_FULL = W_B + 1;           // the accumulators are final
  static constexpr int DRAIN = ACC_FULL + 1;
  static constexpr int NBAR = DRAIN + 1;
  static constexpr int SMEM_FIX = 0;
  static constexpr int SMEM_STREAM = 2 * TILE;
  static constexpr int SMEM_VEC = SMEM_STREAM + NSTAGE * 2 * TILE;   // per stage: lse2[128], dsum[128]
  static constexpr int SMEM_BAR = SMEM_VEC + NSTAGE * 2 * BM * 4;
  static constexpr int SMEM_MISC = SMEM_BAR + NBAR * 8;
  static constexpr int SMEM_USED = SMEM_MISC + 16 + 1024;
  // at least 120 KB, so that one CTA holds an SM (and its whole TMEM)
  static constexpr int SMEM_BYTES = SMEM_USED > 122880 ? SMEM_USED : 122880;
};

struct Params {
  const float* lse;         // forward LSE [B, H, Sq] (natural log)
  float* lse2;              // workspace: LSE * log2(e), [B * H, Sq_pad], +inf past Sq
  float* dsum;              // workspace: rowsum(dO * O), [B * H, Sq_pad], 0 past Sq
  const uint8_t* o;
  const uint8_t* dout;
  uint8_t* dq;
  uint8_t* dk;
  uint8_t* dv;
  long long q_bs, q_hs, q_rs;   // byte strides (batch, head, row) of q-shaped tensors
  long long k_bs, k_hs, k_rs;   // of k-shaped tensors
  int B, H, Sq, Sk, Sq_pad, tq, tk;
  int causal, bhsd;
  float scale, scale_log2;
  unsigned long long wait_limit_ns;
  float* dq_acc;            // non-deterministic variant: fp32 dQ accumulator [B * H, Sq_pad, D]
};

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
               : "memory");
}

__device__ __forceinline__ float2 unpack2(uint32_t w, bool bf16) {
  if (bf16) {
    __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&w);
    return __bfloat1622float2(v);
  }
  __half2 v = *reinterpret_cast<__half2*>(&w);
  return __half22float2(v);
}

// ----------------------------------------------------------------------------- 1. per-row D and LSE * log2 e

// One warp per (padded) row: D_i = sum_d dO_id O_id in fp32.
template <int D, bool BF16>
__global__ void __launch_bounds__(256) prep_kernel(const __grid_constant__ Params p) {
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const long long total = (long long)p.B * p.H * p.Sq_pad;
  if (row >= total) return;
  const int bh = (int)(row / p.Sq_pad);
  const int i = (int)(row - (long long)bh * p.Sq_pad);
  const int b = bh / p.H, h = bh - b * p.H;
  float lse2 = INFINITY, d = 0.f;
  if (i < p.Sq) {
    const size_t off = (size_t)b * p.q_bs + (size_t)h * p.q_hs + (size_t)i * p.q_rs;
    constexpr int PER = D / 32;   // elements per lane: 4 (D = 128) or 2 (D = 64)
    const uint32_t* o32 = reinterpret_cast<const uint32_t*>(p.o + off) + lane * (PER / 2);
    const uint32_t* d32 = reinterpret_cast<const uint32_t*>(p.dout + off) + lane * (PER / 2);
#pragma unroll
    for (int e = 0; e < PER / 2; ++e) {
      const float2 a = unpack2(o32[e], BF16), g = unpack2(d32[e], BF16);
      d = fmaf(a.x, g.x, d);
      d = fmaf(a.y, g.y, d);
    }
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) d += __shfl_xor_sync(0xffffffffu, d, s);
    lse2 = p.lse[(size_t)bh * p.Sq + i] * 1.4426950408889634074f;
  }
  if (lane == 0) {
    p.lse2[row] = lse2;
    p.dsum[row] = d;
  }
}

// ----------------------------------------------------------------------------- shared pieces

// 128 x 64-column TMA boxes of one 128-row tile (rows s0 .. s0 + 127 of head h, batch b).
__device__ __forceinline__ void load_tile(uint32_t dst, const CUtensorMap* map, uint32_t bar, int nbox, int bhsd,
                                          int s0, int h, int b) {
  for (int bx = 0; bx < nbox; ++bx)
    tma_load_4d(dst + bx * BOX_BYTES, map, bar, bx * 64, bhsd ? s0 : h, bhsd ? h : s0, b);
}

// TMEM column of the 16-bit P^T / dS^T words of queries [16 kk, 16 kk + 16) of
// a 128-query step: group g packs its 64 queries into columns [64 g, 64 g + 32).
__device__ __forceinline__ uint32_t packed_col(int kk) { return (uint32_t)((kk >> 2) * 64 + (kk & 3) * 8); }

// ----------------------------------------------------------------------------- 2. dK, dV

template <int D, bool BF16>
__global__ void __launch_bounds__(THREADS, 1)
    dkdv_kernel(const __grid_constant__ Params p, const __grid_constant__ CUtensorMap tmQ,
                const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                const __grid_constant__ CUtensorMap tmDO) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sFix = smem_u32(smem + C::SMEM_FIX);         // K tile, V tile
  const uint32_t sStr = smem_u32(smem + C::SMEM_STREAM);      // per stage: Q_i, dO_i
  const float* sVec = reinterpret_cast<const float*>(smem + C::SMEM_VEC);
  const uint32_t bars = smem_u32(smem + C::SMEM_BAR);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::SMEM_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::SMEM_MISC + 4);
  auto bar = [&](int i) -> uint32_t { return bars + 8u * (uint32_t)i; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t limit = p.wait_limit_ns;

  // longest first: the first key tiles see the most query tiles (causal)
  const int bhs = p.B * p.H;
  const int kt = blockIdx.x / bhs;
  const int bh = blockIdx.x - kt * bhs;
  const int b = bh / p.H, h = bh - b * p.H;
  const int k0 = kt * BN;
  const int i_begin = p.causal ? kt : 0;     // query tiles with a row >= some key of this tile
  const int i_end = p.tq;
  const int nq = max(0, i_end - i_begin);

  if (threadIdx.x == 0) {
    mbar_init(bar(C::IN_FULL), 1);
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(bar(C::ST_FULL + s), 1);
      mbar_init(bar(C::ST_EMPTY + s), 1);
    }
    mbar_init(bar(C::S_FULL), 1);
    mbar_init(bar(C::DP_FULL), 1);
    mbar_init(bar(C::W_A), 2 * BM);
    mbar_init(bar(C::W_B), 2 * BM);
    mbar_init(bar(C::ACC_FULL), 1);
    mbar_init(bar(C::DRAIN), 1);
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
  constexpr uint32_t IDESC_ST = idesc_f16(BM, BM, FMT, 0);    // 128 keys x 128 queries, both K-major
  constexpr uint32_t IDESC_ACC = idesc_f16(BM, D, FMT, 1);    // 128 keys x D, A in TMEM, B MN-major

  if (warp == LOAD_WARP) {
    if (lane == 0 && nq > 0) {
      bool ok = true;
      mbar_arrive_expect_tx(bar(C::IN_FULL), 2 * C::TILE);
      load_tile(sFix, &tmK, bar(C::IN_FULL), C::NBOX, p.bhsd, k0, h, b);
      load_tile(sFix + C::TILE, &tmV, bar(C::IN_FULL), C::NBOX, p.bhsd, k0, h, b);
      uint32_t issued = 0;
      for (int i = i_begin; i < i_end && ok; ++i, ++issued) {
        const uint32_t st = issued % NSTAGE;
        ok = wait_bar1(bar(C::ST_EMPTY + st), ((issued / NSTAGE) & 1u) ^ 1u, abort_flag, limit);
        if (!ok) break;
        mbar_arrive_expect_tx(bar(C::ST_FULL + st), 2 * C::TILE + 2 * BM * 4);
        const uint32_t dst = sStr + st * 2 * C::TILE;
        load_tile(dst, &tmQ, bar(C::ST_FULL + st), C::NBOX, p.bhsd, i * BM, h, b);
        load_tile(dst + C::TILE, &tmDO, bar(C::ST_FULL + st), C::NBOX, p.bhsd, i * BM, h, b);
        const size_t vo = (size_t)bh * p.Sq_pad + (size_t)i * BM;
        const uint32_t vdst = smem_u32(sVec + st * 2 * BM);
        bulk_load(vdst, p.lse2 + vo, BM * 4, bar(C::ST_FULL + st));
        bulk_load(vdst + BM * 4, p.dsum + vo, BM * 4, bar(C::ST_FULL + st));
      }
      // drain: every load issued has landed
      drain_wait(bar(C::IN_FULL), 0, limit);
      const uint32_t first = issued > (uint32_t)NSTAGE ? issued - NSTAGE : 0u;
      for (uint32_t c = first; c < issued; ++c) drain_wait(bar(C::ST_FULL + c % NSTAGE), (c / NSTAGE) & 1u, limit);
    }
    __syncwarp();
  } else if (warp == MMA_WARP) {
    if (nq > 0) {
      bool ok = wait_bar(bar(C::IN_FULL), 0, abort_flag, limit);
      const uint64_t dK0 = sdesc(sFix, 16, 1024), dV0k = sdesc(sFix + C::TILE, 16, 1024);
      const uint64_t dStr = sdesc(sStr, 16, 1024);          // K-major view of a streamed tile
      const uint64_t dStrMN = sdesc(sStr, BOX_BYTES, 1024);  // MN-major view
      constexpr uint32_t TILE16 = C::TILE >> 4;
      const uint32_t tST = tmem, tDPT = tmem + BM, tDV = tmem + 2 * BM, tDK = tmem + 2 * BM + D;
      auto st_products = [&](uint32_t n) {     // S^T(n) = K Q_n^T
        const uint64_t q_k = dStr + (uint64_t)((n % NSTAGE) * 2 * TILE16);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (uint32_t)((kk >> 2) * (BOX_BYTES >> 4) + (kk & 3) * 2);
            mma_ss(tST, dK0 + off, q_k + off, IDESC_ST, kk > 0 ? 1u : 0u);
          }
        }
        __syncwarp();
      };
      auto dpt_products = [&](uint32_t n) {    // dP^T(n) = V dO_n^T
        const uint64_t do_k = dStr + (uint64_t)((n % NSTAGE) * 2 * TILE16 + TILE16);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (uint32_t)((kk >> 2) * (BOX_BYTES >> 4) + (kk & 3) * 2);
            mma_ss(tDPT, dV0k + off, do_k + off, IDESC_ST, kk > 0 ? 1u : 0u);
          }
        }
        __syncwarp();
      };
      // Order of the tensor work: S^T(0), dP^T(0), then per step n
      //   dV(n), S^T(n+1), dK(n), dP^T(n+1)
      // so that the compute warps work out P^T(n+1) from S^T(n+1) while
      // dK(n) and dP^T(n+1) run, and dS^T(n+1) while dV(n+1) and S^T(n+2) run.
      // S^T(n+1) overwrites P^T(n) and dP^T(n+1) overwrites dS^T(n) only
      // after the products that read them (tcgen05 MMAs run in issue order).
      if (ok) ok = wait_bar(bar(C::ST_FULL), 0, abort_flag, limit);
      if (ok) {
        tc_fence_after();
        st_products(0);
        tc_commit_elect(bar(C::S_FULL));
        dpt_products(0);
        tc_commit_elect(bar(C::DP_FULL));
      }
      for (uint32_t n = 0; n < (uint32_t)nq && ok; ++n) {
        const uint32_t st = n % NSTAGE;
        const uint64_t q_mn = dStrMN + (uint64_t)(st * 2 * TILE16);
        const uint64_t do_mn = q_mn + TILE16;
        ok = wait_bar(bar(C::W_A), n & 1u, abort_flag, limit);     // P^T(n) written
        if (!ok) break;
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < BM / 16; ++kk)    // dV += P^T dO_n  (P^T: 8 packed columns per 16 queries)
            mma_ts(tDV, tST + packed_col(kk), do_mn + (uint64_t)(kk * 128), IDESC_ACC, (n > 0 || kk > 0) ? 1u : 0u);
        }
        __syncwarp();
        const bool more = n + 1 < (uint32_t)nq;
        if (more) {
          ok = wait_bar(bar(C::ST_FULL + (n + 1) % NSTAGE), ((n + 1) / NSTAGE) & 1u, abort_flag, limit);
          if (!ok) break;
          tc_fence_after();
          st_products(n + 1);
          tc_commit_elect(bar(C::S_FULL));
        }
        ok = wait_bar(bar(C::W_B), n & 1u, abort_flag, limit);     // dS^T(n) written
        if (!ok) break;
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < BM / 16; ++kk)    // dK += dS^T Q_n
            mma_ts(tDK, tDPT + packed_col(kk), q_mn + (uint64_t)(kk * 128), IDESC_ACC, (n > 0 || kk > 0) ? 1u : 0u);
        }
        __syncwarp();
        tc_commit_elect(bar(C::ST_EMPTY + st));
        if (more) {
          dpt_products(n + 1);
          tc_commit_elect(bar(C::DP_FULL));
        }
      }
      if (ok) tc_commit_elect(bar(C::ACC_FULL));
      tc_commit_elect(bar(C::DRAIN));
      if (lane == 0) drain_wait(bar(C::DRAIN), 0, limit);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- compute warpgroup: one thread per key
    const int quad = warp & 3, grp = warp >> 2;
    const int rit = quad * 32 + lane;
    const int key = k0 + rit;
    const uint32_t lane_bits = (uint32_t)(quad * 32) << 16;
    const uint32_t tST = tmem + lane_bits, tDPT = tmem + lane_bits + BM;
    const uint32_t tDV = tmem + lane_bits + 2 * BM, tDK = tmem + lane_bits + 2 * BM + D;
    const float c = p.scale_log2;
    bool ok = true;
    uint32_t n = 0;
    for (int i = i_begin; i < i_end && ok; ++i, ++n) {
      const uint32_t st = n % NSTAGE;
      // the stage's query vectors came by a bulk copy: observe its completion
      ok = wait_bar(bar(C::ST_FULL + st), (n / NSTAGE) & 1u, abort_flag, limit);
      if (!ok) break;
      const float* vl = sVec + st * 2 * BM;        // lse2 of the tile's queries
      const float* vd = vl + BM;                   // their D
      const int q0 = i * BM;
      // causal: query q sees this key iff q >= key; only tiles that reach
      // below the key need the test
      const bool masked = p.causal && (q0 < k0 + BM - 1);
      // ---- phase A: P^T = 2^(s c - lse2) from S^T, packed to the input dtype
      // (phase B takes P from these packed words: it is the P the tile
      // products use, and half the registers of an fp32 copy)
      // the group's lse2 values are read before the wait: their shared-memory
      // latency then overlaps the wait instead of following it
      float4 lv4[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) lv4[i] = *reinterpret_cast<const float4*>(vl + grp * 64 + 4 * i);
      ok = wait_bar(bar(C::S_FULL), n & 1u, abort_flag, limit);
      if (!ok) break;
      tc_fence_after();
      uint32_t pk[32];
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        const int col = grp * 64 + ch * 32;          // query columns [col, col + 32)
        uint32_t sv[32];
        tmem_ld32(tST + col, sv);
        tmem_wait_ld();
        reg_fence(sv);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int qa = col + 2 * e;
          const float4 l4 = lv4[ch * 8 + (e >> 1)];
          const float la = (qa & 2) ? l4.z : l4.x, lb = (qa & 2) ? l4.w : l4.y;
          float pa = ex2(fmaf(__uint_as_float(sv[2 * e]), c, -la));
          float pb = ex2(fmaf(__uint_as_float(sv[2 * e + 1]), c, -lb));
          if (masked) {
            if (q0 + qa < key) pa = 0.f;
            if (q0 + qa + 1 < key) pb = 0.f;
          }
          pk[ch * 16 + e] = pack2<BF16>(pa, pb);
        }
      }
      // P^T of group g goes over the first half of the S^T columns it read
      // itself, [64 g, 64 g + 32): no other thread reads them.
      tmem_st32(tST + grp * 64, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(C::W_A));
      // ---- phase B: dS^T = P^T (dP^T - D)
      float4 dv4[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) dv4[i] = *reinterpret_cast<const float4*>(vd + grp * 64 + 4 * i);
      ok = wait_bar(bar(C::DP_FULL), n & 1u, abort_flag, limit);
      if (!ok) break;
      tc_fence_after();
      uint32_t pg[32];
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        const int col = grp * 64 + ch * 32;
        uint32_t dp[32];
        tmem_ld32(tDPT + col, dp);
        tmem_wait_ld();
        reg_fence(dp);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int qa = col + 2 * e;
          const float4 d4 = dv4[ch * 8 + (e >> 1)];
          const float da = (qa & 2) ? d4.z : d4.x, db = (qa & 2) ? d4.w : d4.y;
          const float2 pp = unpack2(pk[ch * 16 + e], BF16);
          pg[ch * 16 + e] = pack2<BF16>(pp.x * (__uint_as_float(dp[2 * e]) - da), pp.y * (__uint_as_float(dp[2 * e + 1]) - db));
        }
      }
      tmem_st32(tDPT + grp * 64, pg);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(C::W_B));
    }
    // ---------------------------------------------------------------- epilogue: dV and scale * dK rows
    const bool store = key < p.Sk;
    uint8_t* dvrow = p.dv + (size_t)b * p.k_bs + (size_t)h * p.k_hs + (size_t)key * p.k_rs;
    uint8_t* dkrow = p.dk + (size_t)b * p.k_bs + (size_t)h * p.k_hs + (size_t)key * p.k_rs;
    // group 0 stores the dV row, group 1 the dK row
    uint8_t* dst = grp ? dkrow : dvrow;
    if (nq == 0) {
      // no query sees this key: its gradients are zero
      if (store) {
#pragma unroll
        for (int e = 0; e < D * 2 / 16; ++e) reinterpret_cast<uint4*>(dst)[e] = make_uint4(0, 0, 0, 0);
      }
    } else if (ok) {
      ok = wait_bar(bar(C::ACC_FULL), 0, abort_flag, limit);
      if (ok) {
        tc_fence_after();
        {
          const uint32_t src = grp ? tDK : tDV;
          const float f = grp ? p.scale : 1.f;
#pragma unroll
          for (int q4 = 0; q4 < D / 32; ++q4) {
            uint32_t r[32];
            tmem_ld32(src + q4 * 32, r);
            tmem_wait_ld();
            reg_fence(r);
            uint32_t w[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) w[e] = pack2<BF16>(__uint_as_float(r[2 * e]) * f, __uint_as_float(r[2 * e + 1]) * f);
            if (store) {
#pragma unroll
              for (int e = 0; e < 4; ++e)
                reinterpret_cast<uint4*>(dst + q4 * 64)[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
            }
          }
        }
      }
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

// ----------------------------------------------------------------------------- 3. dQ

template <int D, bool BF16>
__global__ void __launch_bounds__(THREADS, 1)
    dq_kernel(const __grid_constant__ Params p, const __grid_constant__ CUtensorMap tmQ,
              const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
              const __grid_constant__ CUtensorMap tmDO) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sFix = smem_u32(smem + C::SMEM_FIX);         // Q tile, dO tile
  const uint32_t sStr = smem_u32(smem + C::SMEM_STREAM);      // per stage: K_j, V_j
  const uint32_t bars = smem_u32(smem + C::SMEM_BAR);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::SMEM_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::SMEM_MISC + 4);
  auto bar = [&](int i) -> uint32_t { return bars + 8u * (uint32_t)i; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t limit = p.wait_limit_ns;

  // longest first: causal, the last query tiles see the most keys
  const int bhs = p.B * p.H;
  const int lvl = blockIdx.x / bhs;
  const int bh = blockIdx.x - lvl * bhs;
  const int qt = p.causal ? p.tq - 1 - lvl : lvl;
  const int b = bh / p.H, h = bh - b * p.H;
  const int q0 = qt * BM;
  int nk = p.tk;
  if (p.causal) {
    const int last_row = min(q0 + BM - 1, p.Sq - 1);
    nk = min(last_row, p.Sk - 1) / BN + 1;
  }

  if (threadIdx.x == 0) {
    mbar_init(bar(C::IN_FULL), 1);
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(bar(C::ST_FULL + s), 1);
      mbar_init(bar(C::ST_EMPTY + s), 1);
    }
    mbar_init(bar(C::S_FULL), 1);
    mbar_init(bar(C::DP_FULL), 1);
    mbar_init(bar(C::RD_A), 2 * BM);
    mbar_init(bar(C::W_A), 2 * BM);
    mbar_init(bar(C::W_B), 2 * BM);
    mbar_init(bar(C::ACC_FULL), 1);
    mbar_init(bar(C::DRAIN), 1);
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
  constexpr uint32_t IDESC_S = idesc_f16(BM, BN, FMT, 0);     // 128 queries x 128 keys, both K-major
  constexpr uint32_t IDESC_ACC = idesc_f16(BM, D, FMT, 1);    // 128 queries x D, A in TMEM, B MN-major

  if (warp == LOAD_WARP) {
    if (lane == 0) {
      bool ok = true;
      mbar_arrive_expect_tx(bar(C::IN_FULL), 2 * C::TILE);
      load_tile(sFix, &tmQ, bar(C::IN_FULL), C::NBOX, p.bhsd, q0, h, b);
      load_tile(sFix + C::TILE, &tmDO, bar(C::IN_FULL), C::NBOX, p.bhsd, q0, h, b);
      uint32_t issued = 0;
      for (int j = 0; j < nk && ok; ++j, ++issued) {
        const uint32_t st = issued % NSTAGE;
        ok = wait_bar1(bar(C::ST_EMPTY + st), ((issued / NSTAGE) & 1u) ^ 1u, abort_flag, limit);
        if (!ok) break;
        mbar_arrive_expect_tx(bar(C::ST_FULL + st), 2 * C::TILE);
        const uint32_t dst = sStr + st * 2 * C::TILE;
        load_tile(dst, &tmK, bar(C::ST_FULL + st), C::NBOX, p.bhsd, j * BN, h, b);
        load_tile(dst + C::TILE, &tmV, bar(C::ST_FULL + st), C::NBOX, p.bhsd, j * BN, h, b);
      }
      drain_wait(bar(C::IN_FULL), 0, limit);
      const uint32_t first = issued > (uint32_t)NSTAGE ? issued - NSTAGE : 0u;
      for (uint32_t c = first; c < issued; ++c) drain_wait(bar(C::ST_FULL + c % NSTAGE), (c / NSTAGE) & 1u, limit);
    }
    __syncwarp();
  } else if (warp == MMA_WARP) {
    bool ok = wait_bar(bar(C::IN_FULL), 0, abort_flag, limit);
    const uint64_t dQd = sdesc(sFix, 16, 1024), dDOd = sdesc(sFix + C::TILE, 16, 1024);
    const uint64_t dStr = sdesc(sStr, 16, 1024);
    const uint64_t dStrMN = sdesc(sStr, BOX_BYTES, 1024);
    constexpr uint32_t TILE16 = C::TILE >> 4;
    // TMEM: S in two buffers (columns [0, 128) and [256 + D, 384 + D)), dP,
    // dQ.  S(j + 1) and dP(j + 1) are issued as soon as both compute groups
    // have read S(j) and dP(j), so they run while dS(j) is being written and
    // dQ += dS(j) K_j follows; S(j + 1) goes to the other buffer, away from
    // dS(j).
    const uint32_t tDP = tmem + BN, tDQ = tmem + 2 * BN;
    auto s_buf = [&](uint32_t j) -> uint32_t { return (j & 1u) ? tmem + 2 * BN + D : tmem; };
    auto s_dp_products = [&](uint32_t j) {
      const uint64_t k_k = dStr + (uint64_t)((j % NSTAGE) * 2 * TILE16);
      const uint64_t v_k = k_k + TILE16;
      const uint32_t tS = s_buf(j);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {   // S = Q K_j^T
          const uint32_t off = (uint32_t)((kk >> 2) * (BOX_BYTES >> 4) + (kk & 3) * 2);
          mma_ss(tS, dQd + off, k_k + off, IDESC_S, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {   // dP = dO V_j^T
          const uint32_t off = (uint32_t)((kk >> 2) * (BOX_BYTES >> 4) + (kk & 3) * 2);
          mma_ss(tDP, dDOd + off, v_k + off, IDESC_S, kk > 0 ? 1u : 0u);
        }
      }
      __syncwarp();
    };
    if (ok) ok = wait_bar(bar(C::ST_FULL), 0, abort_flag, limit);
    if (ok) {
      tc_fence_after();
      s_dp_products(0);
      tc_commit_elect(bar(C::S_FULL));
    }
    for (uint32_t j = 0; j < (uint32_t)nk && ok; ++j) {
      const uint32_t st = j % NSTAGE;
      ok = wait_bar(bar(C::RD_A), j & 1u, abort_flag, limit);     // S(j), dP(j) read
      if (!ok) break;
      if (j + 1 < (uint32_t)nk) {
        ok = wait_bar(bar(C::ST_FULL + (j + 1) % NSTAGE), ((j + 1) / NSTAGE) & 1u, abort_flag, limit);
        if (!ok) break;
        tc_fence_after();
        s_dp_products(j + 1);
        tc_commit_elect(bar(C::S_FULL));
      }
      ok = wait_bar(bar(C::W_A), j & 1u, abort_flag, limit);      // dS(j) written
      if (!ok) break;
      tc_fence_after();
      const uint64_t k_mn = dStrMN + (uint64_t)(st * 2 * TILE16);
      const uint32_t tS = s_buf(j);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)    // dQ += dS K_j
          mma_ts(tDQ, tS + packed_col(kk), k_mn + (uint64_t)(kk * 128), IDESC_ACC, (j > 0 || kk > 0) ? 1u : 0u);
      }
      __syncwarp();
      tc_commit_elect(bar(C::ST_EMPTY + st));
    }
    if (ok) tc_commit_elect(bar(C::ACC_FULL));
    tc_commit_elect(bar(C::DRAIN));
    if (lane == 0) drain_wait(bar(C::DRAIN), 0, limit);
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- compute warpgroup: one thread per query row
    const int quad = warp & 3, grp = warp >> 2;
    const int rit = quad * 32 + lane;
    const int row = q0 + rit;
    const uint32_t lane_bits = (uint32_t)(quad * 32) << 16;
    const uint32_t tDP = tmem + lane_bits + BN, tDQ = tmem + lane_bits + 2 * BN;
    const float c = p.scale_log2;
    const size_t vo = (size_t)bh * p.Sq_pad + (size_t)row;     // padded: in bounds for every row of the tile
    const float lse2 = p.lse2[vo];
    const float dsum = p.dsum[vo];
    bool ok = true;
    for (int j = 0; j < nk && ok; ++j) {
      ok = wait_bar(bar(C::S_FULL), (uint32_t)j & 1u, abort_flag, limit);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tS = tmem + lane_bits + ((j & 1) ? 2 * BN + D : 0);   // this step's S buffer
      const int c0 = j * BN;
      const bool masked = (c0 + BN > p.Sk) || (p.causal && c0 + BN - 1 > q0);
      int lim = p.Sk - 1 - c0;                 // last key (relative) this row sees
      if (p.causal) lim = min(lim, row - c0);
      // Read this group's half of S and dP first, then tell the MMA warp:
      // S(j + 1) and dP(j + 1) run while the exponentials below are computed.
      uint32_t sv[64], dp[64];
      tmem_ld32(tS + grp * 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
      tmem_ld32(tS + grp * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
      tmem_ld32(tDP + grp * 64, *reinterpret_cast<uint32_t(*)[32]>(&dp[0]));
      tmem_ld32(tDP + grp * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&dp[32]));
      tmem_wait_ld();
      reg_fence(sv);
      reg_fence(dp);
      tc_fence_before();
      mbar_arrive(bar(C::RD_A));
      uint32_t pd[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int ka = grp * 64 + 2 * e;       // key column within the tile
        float pa = ex2(fmaf(__uint_as_float(sv[2 * e]), c, -lse2));
        float pb = ex2(fmaf(__uint_as_float(sv[2 * e + 1]), c, -lse2));
        if (masked) {
          if (ka > lim) pa = 0.f;
          if (ka + 1 > lim) pb = 0.f;
        }
        pd[e] = pack2<BF16>(pa * (__uint_as_float(dp[2 * e]) - dsum), pb * (__uint_as_float(dp[2 * e + 1]) - dsum));
      }
      // dS of group g goes over the first half of the S columns it read
      // itself, [64 g, 64 g + 32): no other thread reads them.
      tmem_st32(tS + grp * 64, pd);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(C::W_A));
    }
    if (ok) ok = wait_bar(bar(C::ACC_FULL), 0, abort_flag, limit);
    if (ok) {
      tc_fence_after();
      uint8_t* dqrow = p.dq + (size_t)b * p.q_bs + (size_t)h * p.q_hs + (size_t)row * p.q_rs;
      // group g stores dQ columns [g D/2, (g + 1) D/2)
#pragma unroll
      for (int q2 = 0; q2 < D / 64; ++q2) {
        const int q4 = grp * (D / 64) + q2;
        uint32_t r[32];
        tmem_ld32(tDQ + q4 * 32, r);
        tmem_wait_ld();
        reg_fence(r);
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          w[e] = pack2<BF16>(__uint_as_float(r[2 * e]) * p.scale, __uint_as_float(r[2 * e + 1]) * p.scale);
        if (row < p.Sq) {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            reinterpret_cast<uint4*>(dqrow + q4 * 64)[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
        }
      }
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

}  // namespace bwd
}  // namespace fa

// The non-deterministic variant (dQ added across key tiles) shares the prep
// kernel, the parameters and the host checks.
#include "fa_bwd_atomic_impl.cuh"

// ============================================================================= host side (backward)

namespace {

struct BwdConfigured {
  bool done[3][4] = {};
};
BwdConfigured g_bwd_cfg[kMaxDevices];

int64_t bwd_sq_pad(int64_t Sq) { return (Sq + fa::BM - 1) / fa::BM * fa::BM; }

template <int D, bool BF16>
fa_status launch_bwd(fa::bwd::Params& prm, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                     const CUtensorMap& mdo, int dev, cudaStream_t s, int slot) {
  using C = fa::bwd::Cfg<D>;
  auto kdkdv = fa::bwd::dkdv_kernel<D, BF16>;
  auto kdq = fa::bwd::dq_kernel<D, BF16>;
  {
    std::lock_guard<std::mutex> g(g_dev_mu);
    if (!g_bwd_cfg[dev].done[0][slot]) {
      cudaError_t e = cudaFuncSetAttribute(kdkdv, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
      if (e != cudaSuccess) return cuda_fail((int)e);
      e = cudaFuncSetAttribute(kdq, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
      if (e != cudaSuccess) return cuda_fail((int)e);
      g_bwd_cfg[dev].done[0][slot] = true;
    }
  }
  const long long rows = (long long)prm.B * prm.H * prm.Sq_pad;
  fa::bwd::prep_kernel<D, BF16><<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(prm);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail((int)e);
  kdkdv<<<(unsigned)(prm.B * prm.H * prm.tk), fa::bwd::THREADS, C::SMEM_BYTES, s>>>(prm, mq, mk, mv, mdo);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail((int)e);
  kdq<<<(unsigned)(prm.B * prm.H * prm.tq), fa::bwd::THREADS, C::SMEM_BYTES, s>>>(prm, mq, mk, mv, mdo);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail((int)e);
  return FA_OK;
}

}  // namespace

extern "C" {

size_t fa_bwd_workspace_size(int64_t B, int64_t H, int64_t Sq) {
  if (B <= 0 || H <= 0 || Sq <= 0) return 0;
  return (size_t)(2 * B * H * bwd_sq_pad(Sq)) * sizeof(float);
}

}  // extern "C"

namespace {

size_t bwd_atomic_workspace_size(int64_t B, int64_t H, int64_t Sq, int64_t D);

// Validation, tensor maps and parameters shared by fa_bwd and fa_bwd_atomic.
fa_status bwd_impl(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                   void* dq, void* dk, void* dv, int64_t B, int64_t H, int64_t Sq, int64_t Sk, int64_t D,
                   fa_layout layout, int causal, float scale, fa_dtype dtype, void* workspace,
                   size_t workspace_bytes, void* stream, bool atomic) {
  // ---- arguments that need no device
  if (B <= 0 || H <= 0 || Sq < 0 || Sk <= 0 || D <= 0) return FA_ERR_INVALID_ARG;
  if (layout != FA_BSND && layout != FA_BHSD) return FA_ERR_INVALID_ARG;
  if (dtype != FA_FP16 && dtype != FA_BF16) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  const int64_t lim = (int64_t)1 << 30;
  if (B >= lim || H >= lim || Sq >= lim || Sk >= lim || B * H >= lim) return FA_ERR_UNSUPPORTED;
  const int64_t tq = (Sq + fa::BM - 1) / fa::BM, tk = (Sk + fa::BN - 1) / fa::BN;
  if (B * H * tq >= lim || B * H * tk >= lim || B * H * bwd_sq_pad(Sq) >= lim) return FA_ERR_UNSUPPORTED;
  const size_t qbytes = (size_t)(B * H * Sq * D) * 2, kvbytes = (size_t)(B * H * Sk * D) * 2;
  const size_t lbytes = (size_t)(B * H * Sq) * 4;
  if (Sq == 0) {
    // no query rows: no key is seen, so dK = dV = 0 (dQ is empty)
    if (!dk || !dv) return FA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(dk) | reinterpret_cast<uintptr_t>(dv)) & 15u) return FA_ERR_MISALIGNED;
    if (overlaps(dk, kvbytes, dv, kvbytes)) return FA_ERR_ALIAS;
    int dev = 0, sms = 0;
    const void* ptrs[2] = {dk, dv};
    fa_status st = device_checks(ptrs, 2, &dev, &sms);
    if (st != FA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(dk, 0, kvbytes, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(dv, 0, kvbytes, s);
    return e == cudaSuccess ? FA_OK : cuda_fail((int)e);
  }
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv || !workspace) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v) |
       reinterpret_cast<uintptr_t>(o) | reinterpret_cast<uintptr_t>(dout) | reinterpret_cast<uintptr_t>(dq) |
       reinterpret_cast<uintptr_t>(dk) | reinterpret_cast<uintptr_t>(dv) | reinterpret_cast<uintptr_t>(workspace)) &
      15u)
    return FA_ERR_MISALIGNED;
  if (reinterpret_cast<uintptr_t>(lse) & 3u) return FA_ERR_MISALIGNED;
  const size_t wbytes = atomic ? bwd_atomic_workspace_size(B, H, Sq, D) : fa_bwd_workspace_size(B, H, Sq);
  if (workspace_bytes < wbytes) return FA_ERR_INVALID_ARG;
  const void* outs[4] = {dq, dk, dv, workspace};
  const size_t out_bytes[4] = {qbytes, kvbytes, kvbytes, wbytes};
  const void* ins[6] = {q, k, v, o, dout, lse};
  const size_t in_bytes[6] = {qbytes, kvbytes, kvbytes, qbytes, qbytes, lbytes};
  for (int i = 0; i < 4; ++i) {
    for (int j = 0; j < 6; ++j)
      if (overlaps(outs[i], out_bytes[i], ins[j], in_bytes[j])) return FA_ERR_ALIAS;
    for (int j = i + 1; j < 4; ++j)
      if (overlaps(outs[i], out_bytes[i], outs[j], out_bytes[j])) return FA_ERR_ALIAS;
  }

  // ---- device checks
  int dev = 0, sms = 0;
  const void* ptrs[10] = {q, k, v, o, dout, lse, dq, dk, dv, workspace};
  fa_status st = device_checks(ptrs, 10, &dev, &sms);
  if (st != FA_OK) return st;

  CUtensorMap mq, mk, mv, mdo;
  if ((st = make_map(&mq, q, dtype, layout, B, H, Sq, D)) != FA_OK) return st;
  if ((st = make_map(&mk, k, dtype, layout, B, H, Sk, D)) != FA_OK) return st;
  if ((st = make_map(&mv, v, dtype, layout, B, H, Sk, D)) != FA_OK) return st;
  if ((st = make_map(&mdo, dout, dtype, layout, B, H, Sq, D)) != FA_OK) return st;

  fa::bwd::Params prm;
  prm.lse = lse;
  const int64_t sq_pad = bwd_sq_pad(Sq);
  prm.lse2 = static_cast<float*>(workspace);
  prm.dsum = static_cast<float*>(workspace) + B * H * sq_pad;
  prm.o = static_cast<const uint8_t*>(o);
  prm.dout = static_cast<const uint8_t*>(dout);
  prm.dq = static_cast<uint8_t*>(dq);
  prm.dk = static_cast<uint8_t*>(dk);
  prm.dv = static_cast<uint8_t*>(dv);
  if (layout == FA_BHSD) {
    prm.q_rs = D * 2;
    prm.q_hs = Sq * D * 2;
    prm.k_rs = D * 2;
    prm.k_hs = Sk * D * 2;
  } else {
    prm.q_rs = H * D * 2;
    prm.q_hs = D * 2;
    prm.k_rs = H * D * 2;
    prm.k_hs = D * 2;
  }
  prm.q_bs = H * Sq * D * 2;
  prm.k_bs = H * Sk * D * 2;
  prm.B = (int)B;
  prm.H = (int)H;
  prm.Sq = (int)Sq;
  prm.Sk = (int)Sk;
  prm.Sq_pad = (int)sq_pad;
  prm.tq = (int)tq;
  prm.tk = (int)tk;
  prm.causal = causal ? 1 : 0;
  prm.bhsd = layout == FA_BHSD ? 1 : 0;
  prm.scale = scale;
  prm.scale_log2 = (float)((double)scale * 1.4426950408889634074);
  prm.wait_limit_ns = 1000000000ull;
  prm.dq_acc = nullptr;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (atomic) {
    prm.dq_acc = static_cast<float*>(workspace) + 2 * B * H * sq_pad;
    CUtensorMap mq64, mdo64;
    if ((st = make_map(&mq64, q, dtype, layout, B, H, Sq, D, fa::bwda::SUB)) != FA_OK) return st;
    if ((st = make_map(&mdo64, dout, dtype, layout, B, H, Sq, D, fa::bwda::SUB)) != FA_OK) return st;
    if (D == 128)
      return dtype == FA_BF16 ? launch_bwd_atomic<128, true>(prm, mq64, mk, mv, mdo64, dev, s)
                              : launch_bwd_atomic<128, false>(prm, mq64, mk, mv, mdo64, dev, s);
    return dtype == FA_BF16 ? launch_bwd_atomic<64, true>(prm, mq64, mk, mv, mdo64, dev, s)
                            : launch_bwd_atomic<64, false>(prm, mq64, mk, mv, mdo64, dev, s);
  }
  if (D == 128)
    return dtype == FA_BF16 ? launch_bwd<128, true>(prm, mq, mk, mv, mdo, dev, s, 0)
                            : launch_bwd<128, false>(prm, mq, mk, mv, mdo, dev, s, 1);
  return dtype == FA_BF16 ? launch_bwd<64, true>(prm, mq, mk, mv, mdo, dev, s, 2)
                          : launch_bwd<64, false>(prm, mq, mk, mv, mdo, dev, s, 3);
}

size_t bwd_atomic_workspace_size(int64_t B, int64_t H, int64_t Sq, int64_t D) {
  if (B <= 0 || H <= 0 || Sq <= 0 || D <= 0) return 0;
  return (size_t)(B * H * bwd_sq_pad(Sq)) * (size_t)(2 + D) * sizeof(float);
}

}  // namespace

extern "C" {

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                 void* dq, void* dk, void* dv, int64_t B, int64_t H, int64_t Sq, int64_t Sk, int64_t D,
                 fa_layout layout, int causal, float scale, fa_dtype dtype, void* workspace,
                 size_t workspace_bytes, void* stream) {
  return bwd_impl(q, k, v, o, dout, lse, dq, dk, dv, B, H, Sq, Sk, D, layout, causal, scale, dtype, workspace,
                  workspace_bytes, stream, false);
}

size_t fa_bwd_atomic_workspace_size(int64_t B, int64_t H, int64_t Sq, int64_t D) {
  return bwd_atomic_workspace_size(B, H, Sq, D);
}

fa_status fa_bwd_atomic(const void* q, const void* k, const void* v, const void* o, const void* dout,
                        const float* lse, void* dq, void* dk, void* dv, int64_t B, int64_t H, int64_t Sq,
                        int64_t Sk, int64_t D, fa_layout layout, int causal, float scale, fa_dtype dtype,
                        void* workspace, size_t workspace_bytes, void* stream) {
  return bwd_impl(q, k, v, o, dout, lse, dq, dk, dv, B, H, Sq, Sk, D, layout, causal, scale, dtype, workspace,
                  workspace_bytes, stream, true);
}

}  // extern "C"
