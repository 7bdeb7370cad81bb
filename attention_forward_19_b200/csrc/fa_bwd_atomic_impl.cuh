// fa_bwd_atomic_impl.cuh -- the non-deterministic backward pass: dK, dV and dQ
// from one kernel per key tile, dQ added up across key tiles in fp32.
// Included at the end of fa_fwd.cu after fa_bwd_impl.cuh (whose prep kernel,
// parameters and helpers it uses).
//
// Page "catlass FlashAttention template tuning" (hwcomputing.csdn.net/6a0d4681),
// section on the backward: the `deterministic` switch chooses between an
// ordered accumulation and atomic adds, the latter being faster; results then
// differ from run to run by the order of the additions.  The arithmetic is the
// same as fa_bwd's (P = 2^(S c - LSE2), dS = P (dP - D), dV = P^T dO,
// dK = scale dS^T Q, dQ = scale dS K).
//
// One CTA per 128-key tile walks the visible queries in steps of 64 (D = 64 or 128):
//   S^T = K Q_u^T, dP^T = V dO_u^T         (keys on the TMEM lanes, 64 columns each)
//   dV += P^T dO_u, dK += dS^T Q_u         (A from TMEM, as in fa_bwd)
//   dQ_u^T = K^T dS_u^T                    (both operands from shared memory:
//                                           K^T is the K tile read MN-major, dS^T
//                                           is written there by the compute warps)
// TMEM: dV [0,128) | dK [128,256) | S^T [256,320) | dP^T [320,384) |
// dQ^T [384,448) and [448,512) (two buffers).  A warpgroup of its own
// (warps 12-15, one per TMEM lane quadrant) reads each dQ_u^T tile (lanes =
// head-dim index) and adds it to the fp32 accumulator in global memory with
// red.global.add.f32 from registers, one warp instruction per 128 contiguous
// bytes of a query row, while the compute warps go on to the next step's P^T.
// (Staging the tile in shared memory for one 32 KB bulk reduction was 12 %
// slower: two more barriers, a proxy fence and one thread issuing.)  A last
// kernel scales the accumulator and rounds it into dq.  The 64-query step keeps the TMEM budget at 512
// columns; the stream of Q / dO sub-tiles has three stages.
// D = 64: dQ^T = K^T dS^T is still an M = 128 product (the layout the other
// products use): the K tile's region holds two 64-column boxes as at D = 128,
// the second one zeroed, so K^T read MN-major has 128 rows of which the last
// 64 are zero, and so are dQ^T's last 64 TMEM lanes, which are not added.

namespace fa {
namespace bwda {

using bwd::LOAD_WARP;
using bwd::MMA_WARP;
// 16 warps: 0-7 compute, 8 load, 9 MMA, 10-11 idle, 12-15 dQ adders.  The
// launch gives 512 x 128 registers; setmaxnreg raises the compute warpgroups
// to 168 and lowers the other two to 88: 256 x 168 + 256 x 88 = 65536.
constexpr int THREADS_A = 512;
constexpr int ADD_WARP0 = 12;
constexpr int REGS_COMPUTE = 168;
constexpr int REGS_OTHER = 88;
static_assert(256 * REGS_COMPUTE + 256 * REGS_OTHER <= 65536, "register split exceeds the launch");

constexpr int SUB = 64;          // queries per step
constexpr int NST = 3;           // streamed stages (a Q and a dO sub-tile, two vectors)
constexpr int SUB_BOX = SUB * 128;            // one 64-row x 64-element box: 8 KB
constexpr int KT_BYTES = BM * 128 * 2;        // the K tile's region: two 64-column boxes, 32 KB
constexpr int IN_FULL = 0;
constexpr int ST_FULL = 1;
constexpr int ST_EMPTY = ST_FULL + NST;
constexpr int S_FULL = ST_EMPTY + NST;
constexpr int DP_FULL = S_FULL + 1;
constexpr int DQ_FULL = DP_FULL + 1;          // two: dQ^T buffer 0 / 1 complete
constexpr int W_A = DQ_FULL + 2;              // P^T written (256 arrivals)
constexpr int W_B = W_A + 1;                  // dS^T written to TMEM and shared memory (256)
constexpr int RD_C = W_B + 1;                 // two: a dQ^T buffer read (256)
constexpr int ACC_FULL = RD_C + 2;
constexpr int DRAIN = ACC_FULL + 1;
constexpr int NBAR = DRAIN + 1;

template <int DH>
struct ACfg {
  static constexpr int VT_BYTES = BM * DH * 2;                     // the V tile
  static constexpr int SUBT = SUB * DH * 2;                        // a Q or dO sub-tile
  static constexpr int SMEM_FIX = 0;                               // K tile's region, then the V tile
  static constexpr int SMEM_V = KT_BYTES;
  static constexpr int SMEM_STREAM = KT_BYTES + VT_BYTES;          // per stage: Q_u, dO_u sub-tiles
  static constexpr int SMEM_DST = SMEM_STREAM + NST * 2 * SUBT;    // dS^T: 128 keys x 64 queries, 16-bit, swizzled
  static constexpr int SMEM_VEC = SMEM_DST + BM * SUB * 2;         // per stage: lse2[64], dsum[64]
  static constexpr int SMEM_BAR = SMEM_VEC + NST * 2 * SUB * 4;
  static constexpr int SMEM_MISC = SMEM_BAR + NBAR * 8;
  static constexpr int SMEM_USED = SMEM_MISC + 16 + 1024;
  // at least 120 KB, so that one CTA holds an SM (and its whole TMEM)
  static constexpr int SMEM_BYTES = SMEM_USED > 122880 ? SMEM_USED : 122880;
  static_assert(SMEM_DST % 1024 == 0, "the swizzled dS^T tile needs 1024-byte alignment");
  static_assert(SMEM_STREAM % 1024 == 0, "streamed sub-tiles need 1024-byte alignment");
  static_assert(SMEM_BYTES <= 232448, "shared memory of one CTA");
};

constexpr uint32_t COL_DV = 0, COL_DK = 128, COL_ST = 256, COL_DPT = 320, COL_DQ = 384;

// Instruction descriptor (kind::f16) with both operands' majorness given.
__host__ __device__ constexpr uint32_t idesc_ab(int M, int N, uint32_t fmt, uint32_t a_mn, uint32_t b_mn) {
  return (1u << 4) | (fmt << 7) | (fmt << 10) | (a_mn << 15) | (b_mn << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// TMEM column of the 16-bit P^T / dS^T words of queries [16 kk, 16 kk + 16) of
// a 64-query step: group g packs its 32 queries into columns [32 g, 32 g + 16).
__device__ __forceinline__ uint32_t packed_col64(int kk) { return (uint32_t)((kk >> 1) * 32 + (kk & 1) * 8); }

// The 64-row boxes of one Q / dO sub-tile (rows s0 .. s0 + 63 of head h, batch b), one per 64 columns.
template <int DH>
__device__ __forceinline__ void load_sub(uint32_t dst, const CUtensorMap* map, uint32_t bar, int bhsd, int s0, int h,
                                         int b) {
#pragma unroll
  for (int bx = 0; bx < DH / 64; ++bx)
    tma_load_4d(dst + bx * SUB_BOX, map, bar, bx * 64, bhsd ? s0 : h, bhsd ? h : s0, b);
}

template <int DH, bool BF16>
__global__ void __launch_bounds__(THREADS_A, 1)
    dkdvq_kernel(const __grid_constant__ bwd::Params p, const __grid_constant__ CUtensorMap tmQ64,
                 const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 const __grid_constant__ CUtensorMap tmDO64) {
  using A = ACfg<DH>;
  constexpr int SUBT = A::SUBT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sFix = smem_u32(smem + A::SMEM_FIX);
  const uint32_t sStr = smem_u32(smem + A::SMEM_STREAM);
  const uint32_t sDst = smem_u32(smem + A::SMEM_DST);
  const float* sVec = reinterpret_cast<const float*>(smem + A::SMEM_VEC);
  const uint32_t bars = smem_u32(smem + A::SMEM_BAR);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + A::SMEM_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + A::SMEM_MISC + 4);
  auto bar = [&](int i) -> uint32_t { return bars + 8u * (uint32_t)i; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t limit = p.wait_limit_ns;

  // longest first: the first key tiles see the most queries (causal)
  const int bhs = p.B * p.H;
  const int kt = blockIdx.x / bhs;
  const int bh = blockIdx.x - kt * bhs;
  const int b = bh / p.H, h = bh - b * p.H;
  const int k0 = kt * BN;
  const int t64 = (p.Sq + SUB - 1) / SUB;
  const int u_begin = p.causal ? k0 / SUB : 0;      // the first 64-query sub-tile with a row >= k0
  const int nu = max(0, t64 - u_begin);

  if (threadIdx.x == 0) {
    mbar_init(bar(IN_FULL), 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(bar(ST_FULL + s), 1);
      mbar_init(bar(ST_EMPTY + s), 1);
    }
    mbar_init(bar(S_FULL), 1);
    mbar_init(bar(DP_FULL), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(DQ_FULL + i), 1);
      mbar_init(bar(RD_C + i), 4);      // one arrival per adder warp
    }
    mbar_init(bar(W_A), 2 * BM);
    mbar_init(bar(W_B), 2 * BM);
    mbar_init(bar(ACC_FULL), 1);
    mbar_init(bar(DRAIN), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == MMA_WARP) {
    tmem_alloc(smem_u32(tmem_holder), TMEM_COLS);
    tmem_relinquish();
  }
  if constexpr (DH == 64) {
    // the K tile's second 64-column box: zero rows of K^T read MN-major
    if (warp < LOAD_WARP) {
      uint4* z = reinterpret_cast<uint4*>(smem + A::SMEM_FIX + BOX_BYTES);
      for (int i = threadIdx.x; i < BOX_BYTES / 16; i += LOAD_WARP * 32) z[i] = make_uint4(0, 0, 0, 0);
      fence_proxy_async_smem();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  constexpr uint32_t FMT = BF16 ? 1u : 0u;
  constexpr uint32_t IDESC_ST = idesc_ab(BM, SUB, FMT, 0, 0);    // 128 keys x 64 queries, both K-major
  constexpr uint32_t IDESC_ACC = idesc_ab(BM, DH, FMT, 0, 1);    // 128 keys x D, A in TMEM, B MN-major
  constexpr uint32_t IDESC_DQ = idesc_ab(BM, SUB, FMT, 1, 1);    // 128 (D, zero-padded) x 64 queries, MN-major

  if (warp >= LOAD_WARP && warp < ADD_WARP0) {
   asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REGS_OTHER));
   if (warp == LOAD_WARP) {
    if (lane == 0 && nu > 0) {
      bool ok = true;
      mbar_arrive_expect_tx(bar(IN_FULL), 2 * A::VT_BYTES);
      bwd::load_tile(sFix, &tmK, bar(IN_FULL), DH / 64, p.bhsd, k0, h, b);
      bwd::load_tile(sFix + A::SMEM_V, &tmV, bar(IN_FULL), DH / 64, p.bhsd, k0, h, b);
      uint32_t issued = 0;
      for (int u = 0; u < nu && ok; ++u, ++issued) {
        const uint32_t st = issued % NST;
        ok = wait_bar1(bar(ST_EMPTY + st), ((issued / NST) & 1u) ^ 1u, abort_flag, limit);
        if (!ok) break;
        mbar_arrive_expect_tx(bar(ST_FULL + st), 2 * SUBT + 2 * SUB * 4);
        const uint32_t dst = sStr + st * 2 * SUBT;
        const int q0 = (u_begin + u) * SUB;
        load_sub<DH>(dst, &tmQ64, bar(ST_FULL + st), p.bhsd, q0, h, b);
        load_sub<DH>(dst + SUBT, &tmDO64, bar(ST_FULL + st), p.bhsd, q0, h, b);
        const size_t vo = (size_t)bh * p.Sq_pad + (size_t)q0;
        const uint32_t vdst = smem_u32(sVec + st * 2 * SUB);
        bwd::bulk_load(vdst, p.lse2 + vo, SUB * 4, bar(ST_FULL + st));
        bwd::bulk_load(vdst + SUB * 4, p.dsum + vo, SUB * 4, bar(ST_FULL + st));
      }
      drain_wait(bar(IN_FULL), 0, limit);
      const uint32_t first = issued > (uint32_t)NST ? issued - NST : 0u;
      for (uint32_t c = first; c < issued; ++c) drain_wait(bar(ST_FULL + c % NST), (c / NST) & 1u, limit);
    }
    __syncwarp();
   } else if (warp == MMA_WARP) {
    if (nu > 0) {
      bool ok = wait_bar(bar(IN_FULL), 0, abort_flag, limit);
      const uint64_t dKk = sdesc(sFix, 16, 1024), dVk = sdesc(sFix + A::SMEM_V, 16, 1024);
      const uint64_t dKmn = sdesc(sFix, BOX_BYTES, 1024);         // K^T: the K tile read MN-major
      const uint64_t dStrK = sdesc(sStr, 16, 1024);               // a sub-tile, K-major
      const uint64_t dStrMN = sdesc(sStr, SUB_BOX, 1024);         // a sub-tile, MN-major
      const uint64_t dDst = sdesc(sDst, SUB_BOX, 1024);           // dS^T, MN-major (one 64-query group)
      constexpr uint32_t SUBT16 = SUBT >> 4;
      const uint32_t tST = tmem + COL_ST, tDPT = tmem + COL_DPT, tDV = tmem + COL_DV, tDK = tmem + COL_DK;
      auto kmajor_products = [&](uint32_t d_tmem, uint64_t a, uint64_t bsub) {   // 128 x 64 over K = D
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < DH / 16; ++kk) {
            const uint32_t offa = (uint32_t)((kk >> 2) * (BOX_BYTES >> 4) + (kk & 3) * 2);
            const uint32_t offb = (uint32_t)((kk >> 2) * (SUB_BOX >> 4) + (kk & 3) * 2);
            mma_ss(d_tmem, a + offa, bsub + offb, IDESC_ST, kk > 0 ? 1u : 0u);
          }
        }
        __syncwarp();
      };
      auto q_k = [&](uint32_t u) { return dStrK + (uint64_t)((u % NST) * 2 * SUBT16); };
      auto do_k = [&](uint32_t u) { return dStrK + (uint64_t)((u % NST) * 2 * SUBT16 + SUBT16); };
      // Order of the tensor work: S^T(0), dP^T(0), then per step u
      //   dV(u), S^T(u+1), dK(u), dP^T(u+1), dQ^T(u)
      // S^T(u+1) overwrites P^T(u) and dP^T(u+1) overwrites dS^T(u) only after
      // the products that read them (tcgen05 MMAs run in issue order).
      if (ok) ok = wait_bar(bar(ST_FULL), 0, abort_flag, limit);
      if (ok) {
        tc_fence_after();
        kmajor_products(tST, dKk, q_k(0));
        tc_commit_elect(bar(S_FULL));
        kmajor_products(tDPT, dVk, do_k(0));
        tc_commit_elect(bar(DP_FULL));
      }
      for (uint32_t u = 0; u < (uint32_t)nu && ok; ++u) {
        const uint32_t st = u % NST;
        const uint64_t q_mn = dStrMN + (uint64_t)(st * 2 * SUBT16);
        const uint64_t do_mn = q_mn + SUBT16;
        ok = wait_bar(bar(W_A), u & 1u, abort_flag, limit);        // P^T(u) written
        if (!ok) break;
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < SUB / 16; ++kk)   // dV += P^T dO_u
            mma_ts(tDV, tST + packed_col64(kk), do_mn + (uint64_t)(kk * 128), IDESC_ACC, (u > 0 || kk > 0) ? 1u : 0u);
        }
        __syncwarp();
        const bool more = u + 1 < (uint32_t)nu;
        if (more) {
          ok = wait_bar(bar(ST_FULL + (u + 1) % NST), ((u + 1) / NST) & 1u, abort_flag, limit);
          if (!ok) break;
          tc_fence_after();
          kmajor_products(tST, dKk, q_k(u + 1));
          tc_commit_elect(bar(S_FULL));
        }
        ok = wait_bar(bar(W_B), u & 1u, abort_flag, limit);        // dS^T(u) written
        if (!ok) break;
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < SUB / 16; ++kk)   // dK += dS^T Q_u
            mma_ts(tDK, tDPT + packed_col64(kk), q_mn + (uint64_t)(kk * 128), IDESC_ACC, (u > 0 || kk > 0) ? 1u : 0u);
        }
        __syncwarp();
        tc_commit_elect(bar(ST_EMPTY + st));
        if (more) {
          kmajor_products(tDPT, dVk, do_k(u + 1));
          tc_commit_elect(bar(DP_FULL));
        }
        const uint32_t qb = u & 1u;
        if (u >= 2) {                            // the compute warps have read dQ^T(u - 2) from this buffer
          ok = wait_bar(bar(RD_C + qb), ((u >> 1) - 1) & 1u, abort_flag, limit);
          if (!ok) break;
          tc_fence_after();
        }
        const uint32_t tDQ = tmem + COL_DQ + qb * SUB;
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < BM / 16; ++kk)    // dQ^T = K^T dS^T(u)
            mma_ss(tDQ, dKmn + (uint64_t)(kk * 128), dDst + (uint64_t)(kk * 128), IDESC_DQ, kk > 0 ? 1u : 0u);
        }
        __syncwarp();
        tc_commit_elect(bar(DQ_FULL + qb));
      }
      if (ok) tc_commit_elect(bar(ACC_FULL));
      tc_commit_elect(bar(DRAIN));
      if (lane == 0) drain_wait(bar(DRAIN), 0, limit);
    }
    __syncwarp();
   }
  } else if (warp >= ADD_WARP0) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REGS_OTHER));
    // ---------------------------------------------------------------- dQ adders: lane = head-dim index
    // Warp 12 + q reads TMEM lane quadrant (12 + q) % 4 = q of each dQ_v^T tile
    // (head-dim rows, 64 query columns) and adds it to the fp32 accumulator:
    // one warp instruction covers 128 contiguous bytes of one query row.  At
    // D = 64 the lanes 64-127 (zero rows) are read but not added.
    const int quad = warp & 3;
    const int drow = quad * 32 + lane;
    const uint32_t lane_bits = (uint32_t)(quad * 32) << 16;
    float* dq_acc_bh = p.dq_acc + (size_t)bh * p.Sq_pad * DH;
    for (uint32_t v = 0; v < (uint32_t)nu; ++v) {
      if (!wait_bar(bar(DQ_FULL + (v & 1u)), (v >> 1) & 1u, abort_flag, limit)) break;
      tc_fence_after();
      uint32_t r[2][32];
      tmem_ld32(tmem + lane_bits + COL_DQ + (v & 1u) * SUB, r[0]);
      tmem_ld32(tmem + lane_bits + COL_DQ + (v & 1u) * SUB + 32, r[1]);
      tmem_wait_ld();
      reg_fence(r[0]);
      reg_fence(r[1]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(RD_C + (v & 1u)));
      if (drow < DH) {
        float* dst = dq_acc_bh + (size_t)(u_begin + (int)v) * SUB * DH + drow;
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int j = 0; j < 32; ++j) atomicAdd(dst + (size_t)(32 * h + j) * DH, __uint_as_float(r[h][j]));
      }
    }
    __syncwarp();
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REGS_COMPUTE));
    // ---------------------------------------------------------------- compute: one thread per key (phases A, B);
    // group g takes queries [32 g, 32 g + 32) of a step
    const int quad = warp & 3, grp = warp >> 2;
    const int rit = quad * 32 + lane;
    const int key = k0 + rit;
    const bool key_live = key < p.Sk;
    const uint32_t lane_bits = (uint32_t)(quad * 32) << 16;
    const uint32_t tST = tmem + lane_bits + COL_ST, tDPT = tmem + lane_bits + COL_DPT;
    const uint32_t tDV = tmem + lane_bits + COL_DV, tDK = tmem + lane_bits + COL_DK;
    const float c = p.scale_log2;
    bool ok = true;
    for (uint32_t u = 0; u < (uint32_t)nu && ok; ++u) {
      const uint32_t st = u % NST;
      ok = wait_bar(bar(ST_FULL + st), (u / NST) & 1u, abort_flag, limit);   // the vectors came by bulk copy
      if (!ok) break;
      const float* vl = sVec + st * 2 * SUB;
      const float* vd = vl + SUB;
      const int q0 = (u_begin + (int)u) * SUB;
      const bool masked = p.causal && (q0 < k0 + BM - 1);
      // ---- phase A: P^T = 2^(s c - lse2), packed
      ok = wait_bar(bar(S_FULL), u & 1u, abort_flag, limit);
      if (!ok) break;
      tc_fence_after();
      uint32_t pk[16];
      {
        uint32_t sv[32];
        tmem_ld32(tST + grp * 32, sv);
        tmem_wait_ld();
        reg_fence(sv);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int qa = grp * 32 + 2 * e;
          const float2 l2 = *reinterpret_cast<const float2*>(vl + qa);
          float pa = ex2(fmaf(__uint_as_float(sv[2 * e]), c, -l2.x));
          float pb = ex2(fmaf(__uint_as_float(sv[2 * e + 1]), c, -l2.y));
          if (masked) {
            if (q0 + qa < key) pa = 0.f;
            if (q0 + qa + 1 < key) pb = 0.f;
          }
          if (!key_live) pa = pb = 0.f;         // keys past Sk (zero-filled rows) take no weight
          pk[e] = pack2<BF16>(pa, pb);
        }
      }
      // over the first half of this group's own S^T columns: no other thread reads them
      tmem_st16(tST + grp * 32, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(W_A));
      // ---- phase B: dS^T = P^T (dP^T - D), to TMEM (for dK) and to shared memory (for dQ)
      ok = wait_bar(bar(DP_FULL), u & 1u, abort_flag, limit);
      if (!ok) break;
      tc_fence_after();
      uint32_t pg[16];
      {
        uint32_t dp[32];
        tmem_ld32(tDPT + grp * 32, dp);
        tmem_wait_ld();
        reg_fence(dp);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int qa = grp * 32 + 2 * e;
          const float2 d2 = *reinterpret_cast<const float2*>(vd + qa);
          const float2 pp = bwd::unpack2(pk[e], BF16);
          pg[e] = pack2<BF16>(pp.x * (__uint_as_float(dp[2 * e]) - d2.x), pp.y * (__uint_as_float(dp[2 * e + 1]) - d2.y));
        }
      }
      tmem_st16(tDPT + grp * 32, pg);
      if (u >= 1) {                            // dQ^T(u - 1) has finished reading the shared dS^T tile
        ok = wait_bar(bar(DQ_FULL + ((u - 1) & 1u)), ((u - 1) >> 1) & 1u, abort_flag, limit);
        if (!ok) break;
      }
      {
        // row rit of the 128 x 64 tile, 16-byte chunks 4 grp .. 4 grp + 3, 128-byte swizzle
        uint8_t* row = smem + A::SMEM_DST + rit * 128;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int chunk = (grp * 4 + j) ^ (rit & 7);
          *reinterpret_cast<uint4*>(row + chunk * 16) = make_uint4(pg[4 * j], pg[4 * j + 1], pg[4 * j + 2], pg[4 * j + 3]);
        }
      }
      fence_proxy_async_smem();
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(W_B));
    }
    // ---------------------------------------------------------------- epilogue: dV and scale * dK rows
    const bool store = key < p.Sk;
    uint8_t* dvrow = p.dv + (size_t)b * p.k_bs + (size_t)h * p.k_hs + (size_t)key * p.k_rs;
    uint8_t* dkrow = p.dk + (size_t)b * p.k_bs + (size_t)h * p.k_hs + (size_t)key * p.k_rs;
    uint8_t* dst = grp ? dkrow : dvrow;
    if (nu == 0) {
      if (store) {
#pragma unroll
        for (int e = 0; e < DH * 2 / 16; ++e) reinterpret_cast<uint4*>(dst)[e] = make_uint4(0, 0, 0, 0);
      }
    } else if (ok) {
      ok = wait_bar(bar(ACC_FULL), 0, abort_flag, limit);
      if (ok) {
        tc_fence_after();
        const uint32_t src = grp ? tDK : tDV;
        const float f = grp ? p.scale : 1.f;
#pragma unroll
        for (int q4 = 0; q4 < DH / 32; ++q4) {
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
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// dq = scale * accumulator, rounded to the input dtype: one warp per query row, D / 32 columns per lane.
template <int DH, bool BF16>
__global__ void __launch_bounds__(256) dq_convert_kernel(const __grid_constant__ bwd::Params p) {
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const long long total = (long long)p.B * p.H * p.Sq;
  if (row >= total) return;
  const int bh = (int)(row / p.Sq);
  const int i = (int)(row - (long long)bh * p.Sq);
  const int b = bh / p.H, h = bh - b * p.H;
  const float* src = p.dq_acc + ((size_t)bh * p.Sq_pad + i) * DH;
  uint8_t* dst = p.dq + (size_t)b * p.q_bs + (size_t)h * p.q_hs + (size_t)i * p.q_rs;
  if constexpr (DH == 128) {
    const float4 a = *reinterpret_cast<const float4*>(src + lane * 4);
    *reinterpret_cast<uint2*>(dst + lane * 8) = make_uint2(pack2<BF16>(a.x * p.scale, a.y * p.scale),
                                                           pack2<BF16>(a.z * p.scale, a.w * p.scale));
  } else {
    const float2 a = *reinterpret_cast<const float2*>(src + lane * 2);
    *reinterpret_cast<uint32_t*>(dst + lane * 4) = pack2<BF16>(a.x * p.scale, a.y * p.scale);
  }
}

}  // namespace bwda
}  // namespace fa

// ============================================================================= host side (atomic backward)

namespace {

bool g_bwda_configured[kMaxDevices][4];

template <int DH, bool BF16>
fa_status launch_bwd_atomic(fa::bwd::Params& prm, const CUtensorMap& mq64, const CUtensorMap& mk,
                            const CUtensorMap& mv, const CUtensorMap& mdo64, int dev, cudaStream_t s) {
  auto kern = fa::bwda::dkdvq_kernel<DH, BF16>;
  constexpr int smem = fa::bwda::ACfg<DH>::SMEM_BYTES;
  const int slot = (DH == 128 ? 0 : 2) + (BF16 ? 1 : 0);
  {
    std::lock_guard<std::mutex> g(g_dev_mu);
    if (!g_bwda_configured[dev][slot]) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return cuda_fail((int)e);
      g_bwda_configured[dev][slot] = true;
    }
  }
  const long long rows = (long long)prm.B * prm.H * prm.Sq_pad;
  fa::bwd::prep_kernel<DH, BF16><<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(prm);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail((int)e);
  e = cudaMemsetAsync(prm.dq_acc, 0, (size_t)rows * DH * sizeof(float), s);
  if (e != cudaSuccess) return cuda_fail((int)e);
  kern<<<(unsigned)(prm.B * prm.H * prm.tk), fa::bwda::THREADS_A, smem, s>>>(prm, mq64, mk, mv, mdo64);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail((int)e);
  const long long qrows = (long long)prm.B * prm.H * prm.Sq;
  fa::bwda::dq_convert_kernel<DH, BF16><<<(unsigned)((qrows + 7) / 8), 256, 0, s>>>(prm);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail((int)e);
  return FA_OK;
}

}  // namespace
