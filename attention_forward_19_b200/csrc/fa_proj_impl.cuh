// fa_proj_impl.cuh -- the attention output projection Y = O W^T for sm_100a,
// and the attention + projection entry point.  Included at the end of
// fa_fwd.cu (one translation unit with the PTX helpers, the tensor-map
// encoder and the host checks).
//
// Page "catlass FlashAttention template tuning" (hwcomputing.csdn.net/6a0d4681),
// section on graph fusion: the fused operator "FusedAttnProj" is FlashAttention
// followed by the output MatMul (O times the output weight), so that O is not
// written out and read back as a separate operator's input.  Here O of every
// head of a token forms one row of the GEMM's A operand:
//   Y[b, s, n] = sum_{h, d} O[b, s, h, d] * W[n, h * D + d]
// with W in the usual linear-layer layout [E, H * D] (row n = output feature
// n, contiguous over the H * D inputs).
//
// On B200 the projection is its own dense GEMM (2 B S (H D) E flops, as much
// as a third of the attention's at E = H D), so it runs as a separate
// persistent tcgen05 kernel right after the attention kernel on the same
// stream; its A tiles are read straight from the attention's output through
// the same 4-D tensor map (either layout, no reshape or copy), mostly from L2.
//
// Kernel: one CTA per SM, tiles of 256 tokens x 256 features, K in blocks of
// 64 (two 128-row swizzled boxes of O, one 256-row box of W per block) through
// a 3-stage TMA ring; per 16 inputs the MMA warp issues two M = 128, N = 256
// products that share the W box, into the two halves of TMEM (tokens 0-127 and
// 128-255).  Against a 128 x 256 tile this reads a third fewer operand bytes
// per flop (the kernel's operands come mostly from L2, and at 128 x 256 that
// stream was ~94 bytes per SM cycle at full MMA rate).  TMEM then holds one
// tile, so the epilogue (8 warps: token row = TMEM lane, fp32 -> 16-bit) runs
// between tiles.

namespace fa {
namespace proj {

constexpr int TM = 256;           // tokens per tile: two halves of 128 (TMEM lanes)
constexpr int TN = 256;           // output features per tile (TMEM columns per half)
constexpr int TK = 64;            // inputs per k-block: one 128-byte box row
constexpr int NSTAGE = 3;
constexpr int THREADS = 320;      // warps 0-7 epilogue (warp w: half w / 4, lanes of quadrant w % 4), 8 loads, 9 MMA
constexpr int LOAD_WARP = 8;
constexpr int MMA_WARP = 9;
constexpr int A_HALF = 128 * TK * 2;   // 16 KB: one 128-token box
constexpr int A_BYTES = 2 * A_HALF;    // 32 KB
constexpr int B_BYTES = TN * TK * 2;   // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int FULL = 0, EMPTY = NSTAGE, ACC_FULL = 2 * NSTAGE, ACC_EMPTY = ACC_FULL + 1, DRAIN = ACC_EMPTY + 1;
constexpr int NBAR = DRAIN + 1;
constexpr int SMEM_BAR = NSTAGE * STAGE_BYTES;
constexpr int SMEM_MISC = SMEM_BAR + NBAR * 8;
constexpr int SMEM_BYTES = SMEM_MISC + 16 + 1024;

struct Params {
  uint16_t* y;              // [B, S, E]
  int B, H, S, D, E;
  int bhsd;                 // layout of O
  int mt_per_b;             // ceil(S / TM)
  int nt;                   // ceil(E / TN)
  int kb;                   // H * D / TK
  int tiles;                // B * mt_per_b * nt
  unsigned long long wait_limit_ns;
};

template <bool BF16>
__global__ void __launch_bounds__(THREADS, 1)
    proj_kernel(const __grid_constant__ Params p, const __grid_constant__ CUtensorMap tmO,
                const __grid_constant__ CUtensorMap tmW) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bars = smem_u32(smem + SMEM_BAR);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + SMEM_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SMEM_MISC + 4);
  auto bar = [&](int i) -> uint32_t { return bars + 8u * (uint32_t)i; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t limit = p.wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(bar(FULL + s), 1);
      mbar_init(bar(EMPTY + s), 1);
    }
    mbar_init(bar(ACC_FULL), 1);
    mbar_init(bar(ACC_EMPTY), 8);         // one arrival per epilogue warp
    mbar_init(bar(DRAIN), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == MMA_WARP) {
    tmem_alloc(smem_u32(tmem_holder), 2 * TN);     // 512 columns: the two 128-token halves
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int dbox = p.D / TK;              // 64-element boxes per head
  auto tile_coords = [&](int t, int& b, int& s0, int& n0) {
    const int nt_i = t % p.nt;
    const int m = t / p.nt;
    b = m / p.mt_per_b;
    s0 = (m - b * p.mt_per_b) * TM;
    n0 = nt_i * TN;
  };

  if (warp == LOAD_WARP) {
    if (lane == 0) {
      bool ok = true;
      uint32_t issued = 0;
      // The weight is read by every token tile (it should stay in L2); a
      // token tile's O rows are read by the CTAs of its few feature tiles at
      // about the same time and then never again.
      const uint64_t pol_w = l2_policy_evict_last(), pol_o = l2_policy_evict_first();
      for (int t = blockIdx.x; t < p.tiles && ok; t += gridDim.x) {
        int b, s0, n0;
        tile_coords(t, b, s0, n0);
        for (int kb = 0; kb < p.kb; ++kb, ++issued) {
          const uint32_t st = issued % NSTAGE;
          ok = wait_bar1(bar(EMPTY + st), ((issued / NSTAGE) & 1u) ^ 1u, abort_flag, limit);
          if (!ok) break;
          const uint32_t dst = sbase + st * STAGE_BYTES;
          mbar_arrive_expect_tx(bar(FULL + st), STAGE_BYTES);
          const int h = kb / dbox, d0 = (kb - h * dbox) * TK;
          tma_load_4d_hint(dst, &tmO, bar(FULL + st), d0, p.bhsd ? s0 : h, p.bhsd ? h : s0, b, pol_o);
          const int s1 = s0 + 128;            // may lie past S: the box is zero-filled
          tma_load_4d_hint(dst + A_HALF, &tmO, bar(FULL + st), d0, p.bhsd ? s1 : h, p.bhsd ? h : s1, b, pol_o);
          tma_load_4d_hint(dst + A_BYTES, &tmW, bar(FULL + st), kb * TK, n0, 0, 0, pol_w);
        }
      }
      const uint32_t first = issued > (uint32_t)NSTAGE ? issued - NSTAGE : 0u;
      for (uint32_t c = first; c < issued; ++c) drain_wait(bar(FULL + c % NSTAGE), (c / NSTAGE) & 1u, limit);
    }
    __syncwarp();
  } else if (warp == MMA_WARP) {
    constexpr uint32_t FMT = BF16 ? 1u : 0u;
    constexpr uint32_t IDESC = idesc_f16(128, TN, FMT, 0);    // one 128-token half per product
    bool ok = true;
    uint32_t used = 0;
    int i = 0;
    for (int t = blockIdx.x; t < p.tiles && ok; t += gridDim.x, ++i) {
      ok = wait_bar(bar(ACC_EMPTY), ((uint32_t)i & 1u) ^ 1u, abort_flag, limit);   // the last tile is read
      if (!ok) break;
      tc_fence_after();
      for (int kb = 0; kb < p.kb; ++kb, ++used) {
        const uint32_t st = used % NSTAGE;
        ok = wait_bar(bar(FULL + st), (used / NSTAGE) & 1u, abort_flag, limit);
        if (!ok) break;
        tc_fence_after();
        const uint32_t src = sbase + st * STAGE_BYTES;
        const uint64_t da0 = sdesc(src, 16, 1024), da1 = sdesc(src + A_HALF, 16, 1024);
        const uint64_t db = sdesc(src + A_BYTES, 16, 1024);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < TK / 16; ++kk) {
            const uint32_t acc_in = (kb > 0 || kk > 0) ? 1u : 0u;
            mma_ss(tmem, da0 + (uint64_t)(kk * 2), db + (uint64_t)(kk * 2), IDESC, acc_in);
            mma_ss(tmem + TN, da1 + (uint64_t)(kk * 2), db + (uint64_t)(kk * 2), IDESC, acc_in);
          }
        }
        __syncwarp();
        tc_commit_elect(bar(EMPTY + st));
      }
      if (!ok) break;
      tc_commit_elect(bar(ACC_FULL));
    }
    tc_commit_elect(bar(DRAIN));
    if (lane == 0) drain_wait(bar(DRAIN), 0, limit);
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue: thread = token row of the tile
    const int half = warp >> 2, quad = warp & 3;
    const int row = half * 128 + quad * 32 + lane;
    const uint32_t lane_bits = (uint32_t)(quad * 32) << 16;
    bool ok = true;
    int i = 0;
    for (int t = blockIdx.x; t < p.tiles && ok; t += gridDim.x, ++i) {
      int b, s0, n0;
      tile_coords(t, b, s0, n0);
      ok = wait_bar(bar(ACC_FULL), (uint32_t)i & 1u, abort_flag, limit);
      if (!ok) break;
      tc_fence_after();
      const int s = s0 + row;
      uint16_t* yrow = p.y + ((size_t)b * p.S + (size_t)(s < p.S ? s : 0)) * p.E;
#pragma unroll 1
      for (int c = 0; c < TN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_bits + half * TN + c * 32, r);
        tmem_wait_ld();
        reg_fence(r);
        const int n = n0 + c * 32;
        if (s < p.S && n < p.E) {        // E is a multiple of 32: a chunk is all in or all out
          uint4* dst = reinterpret_cast<uint4*>(yrow + n);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 w;
            w.x = pack2<BF16>(__uint_as_float(r[8 * v + 0]), __uint_as_float(r[8 * v + 1]));
            w.y = pack2<BF16>(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3]));
            w.z = pack2<BF16>(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5]));
            w.w = pack2<BF16>(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7]));
            dst[v] = w;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(ACC_EMPTY));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * TN);
  }
}

}  // namespace proj
}  // namespace fa

namespace {

// W [E, K] row-major (K = H * D contiguous), 64 x 256 boxes.  Encoded with two
// unit outer dimensions so that it is read by the same 4-D copy as O.
fa_status make_w_map(CUtensorMap* map, const void* base, fa_dtype dt, int64_t E, int64_t K) {
  int err = 0;
  EncodeTiledFn enc = get_encode_fn(&err);
  if (!enc) return cuda_fail(err);
  const cuuint64_t dims[4] = {(cuuint64_t)K, (cuuint64_t)E, 1, 1};
  const cuuint64_t strides[3] = {(cuuint64_t)K * 2, (cuuint64_t)K * 2 * E, (cuuint64_t)K * 2 * E};
  const cuuint32_t box[4] = {fa::proj::TK, fa::proj::TN, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUtensorMapDataType t =
      dt == FA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUresult r = enc(map, t, 4, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cuda_fail((int)r);
  return FA_OK;
}

bool g_proj_configured[kMaxDevices][2];

// Host checks that need no device, shared by fa_out_proj and fa_fwd_proj.
fa_status proj_host_checks(const void* o, const void* w, const void* y, int64_t B, int64_t H, int64_t S, int64_t D,
                           int64_t E, fa_layout layout, fa_dtype dtype) {
  if (B <= 0 || H <= 0 || S < 0 || D <= 0 || E <= 0) return FA_ERR_INVALID_ARG;
  if (layout != FA_BSND && layout != FA_BHSD) return FA_ERR_INVALID_ARG;
  if (dtype != FA_FP16 && dtype != FA_BF16) return FA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  if (E % 32 != 0) return FA_ERR_UNSUPPORTED;
  const int64_t lim = (int64_t)1 << 30;
  if (B >= lim || H >= lim || S >= lim || E >= lim || B * H >= lim || H * D >= lim) return FA_ERR_UNSUPPORTED;
  const int64_t tiles = B * ((S + fa::proj::TM - 1) / fa::proj::TM) * ((E + fa::proj::TN - 1) / fa::proj::TN);
  if (tiles >= lim) return FA_ERR_UNSUPPORTED;
  if (S == 0) return FA_OK;
  if (!o || !w || !y) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(o) | reinterpret_cast<uintptr_t>(w) | reinterpret_cast<uintptr_t>(y)) & 15u)
    return FA_ERR_MISALIGNED;
  const size_t ob = (size_t)(B * S * H * D) * 2, wb = (size_t)(E * H * D) * 2, yb = (size_t)(B * S * E) * 2;
  if (overlaps(y, yb, o, ob) || overlaps(y, yb, w, wb)) return FA_ERR_ALIAS;
  return FA_OK;
}

fa_status proj_launch(const void* o, const void* w, void* y, int64_t B, int64_t H, int64_t S, int64_t D, int64_t E,
                      fa_layout layout, fa_dtype dtype, void* stream) {
  int dev = 0, sms = 0;
  const void* ptrs[3] = {o, w, y};
  fa_status st = device_checks(ptrs, 3, &dev, &sms);
  if (st != FA_OK) return st;
  CUtensorMap mo, mw;
  if ((st = make_map(&mo, o, dtype, layout, B, H, S, D)) != FA_OK) return st;
  // make_map's boxes are 128 rows x 64 elements: the A tile of one k-block
  if ((st = make_w_map(&mw, w, dtype, E, H * D)) != FA_OK) return st;
  fa::proj::Params prm;
  prm.y = static_cast<uint16_t*>(y);
  prm.B = (int)B;
  prm.H = (int)H;
  prm.S = (int)S;
  prm.D = (int)D;
  prm.E = (int)E;
  prm.bhsd = layout == FA_BHSD ? 1 : 0;
  prm.mt_per_b = (int)((S + fa::proj::TM - 1) / fa::proj::TM);
  prm.nt = (int)((E + fa::proj::TN - 1) / fa::proj::TN);
  prm.kb = (int)(H * D / fa::proj::TK);
  prm.tiles = prm.B * prm.mt_per_b * prm.nt;
  prm.wait_limit_ns = 1000000000ull;
  const int grid = prm.tiles < sms ? prm.tiles : sms;
  const bool bf16 = dtype == FA_BF16;
  auto kern = bf16 ? fa::proj::proj_kernel<true> : fa::proj::proj_kernel<false>;
  {
    std::lock_guard<std::mutex> g(g_dev_mu);
    if (!g_proj_configured[dev][bf16 ? 1 : 0]) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, fa::proj::SMEM_BYTES);
      if (e != cudaSuccess) return cuda_fail((int)e);
      g_proj_configured[dev][bf16 ? 1 : 0] = true;
    }
  }
  kern<<<grid, fa::proj::THREADS, fa::proj::SMEM_BYTES, static_cast<cudaStream_t>(stream)>>>(prm, mo, mw);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail((int)e);
  return FA_OK;
}

}  // namespace

extern "C" {

fa_status fa_out_proj(const void* o, const void* w_o, void* y, int64_t B, int64_t H, int64_t S, int64_t D,
                      int64_t E, fa_layout layout, fa_dtype dtype, void* stream) {
  fa_status st = proj_host_checks(o, w_o, y, B, H, S, D, E, layout, dtype);
  if (st != FA_OK || S == 0) return st;
  return proj_launch(o, w_o, y, B, H, S, D, E, layout, dtype, stream);
}

fa_status fa_fwd_proj(const void* q, const void* k, const void* v, const void* w_o, void* o, float* lse, void* y,
                      int64_t B, int64_t H, int64_t Sq, int64_t Sk, int64_t D, int64_t E, fa_layout layout,
                      int causal, float scale, fa_dtype dtype, void* workspace, size_t workspace_bytes,
                      void* stream) {
  fa_status st = proj_host_checks(o, w_o, y, B, H, Sq, D, E, layout, dtype);
  if (st != FA_OK) return st;
  if (Sq > 0) {
    const size_t yb = (size_t)(B * Sq * E) * 2, qb = (size_t)(B * H * Sq * D) * 2, kb = (size_t)(B * H * Sk * D) * 2;
    const size_t lb = (size_t)(B * H * Sq) * 4;
    if ((q && overlaps(y, yb, q, qb)) || (k && Sk > 0 && overlaps(y, yb, k, kb)) ||
        (v && Sk > 0 && overlaps(y, yb, v, kb)) || (lse && overlaps(y, yb, lse, lb)))
      return FA_ERR_ALIAS;
    if (w_o && (overlaps(w_o, (size_t)(E * H * D) * 2, o, qb) || (lse && overlaps(w_o, (size_t)(E * H * D) * 2, lse, lb))))
      return FA_ERR_ALIAS;
  }
  st = workspace ? fa_fwd_ws(q, k, v, o, lse, B, H, Sq, Sk, D, layout, causal, scale, dtype, workspace,
                             workspace_bytes, stream)
                 : fa_fwd(q, k, v, o, lse, B, H, Sq, Sk, D, layout, causal, scale, dtype, stream);
  if (st != FA_OK || Sq == 0) return st;
  return proj_launch(o, w_o, y, B, H, Sq, D, E, layout, dtype, stream);
}

}  // extern "C"
