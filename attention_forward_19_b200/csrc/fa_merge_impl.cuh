// Merge of partial attention results (O_i, LSE_i) computed over disjoint key
// blocks, for attention split by key ranges (ring / context-parallel
// attention: page "FlashAttention in ops-transformer on Ascend NPU"
// (ai6s.net/6a0d3bfb), section "what else is in the ops-transformer
// repository": ring attention for long sequences; page "64K long-sequence
// FlashAttention" (ai6s.net/6a140d07), section "performance tuning tips",
// multi-card parallelism: each card holds 8K of a 64K sequence).
//
// With a row's partials normalised over their own key blocks, the result over
// the union of the blocks is the online-normalisation update of page
// "FlashAttention: long-text inference without running out of memory"
// (ai6s.net/6a0d42d8), section on tiling and online normalisation (the running
// max and sum), taken one whole block at a time:
//   LSE = log(exp(LSE_a) + exp(LSE_b))
//   O   = exp(LSE_a - LSE) O_a + exp(LSE_b - LSE) O_b
// The running result is kept in fp32; the last merge writes O rounded to the
// 16-bit input type.  A row whose LSE is -inf (no visible key) has weight 0.
//
// Included at the end of fa_fwd.cu (it uses that file's host helpers).

namespace fa {
namespace merge {

constexpr int THREADS = 256;
constexpr int VEC = 8;   // elements of a row per thread (16 bytes of 16-bit, 32 of fp32)

struct Params {
  const uint16_t* o_part;   // [rows, D] 16-bit
  const float* lse_part;    // [B, H, S]
  float* o_acc;             // [rows, D] fp32, read when HAS_ACC, written unless FINAL
  float* lse_acc;
  uint16_t* o_out;          // [rows, D] 16-bit, written when FINAL
  float* lse_out;
  long long rows;           // B * H * S, in the tensor's memory order
  int H, S, D;
  int bhsd;
};

__device__ __forceinline__ float to_f32(uint16_t x, bool bf16) {
  return bf16 ? __bfloat162float(__ushort_as_bfloat16(x)) : __half2float(__ushort_as_half(x));
}
__device__ __forceinline__ uint16_t from_f32(float x, bool bf16) {
  return bf16 ? __bfloat16_as_ushort(__float2bfloat16_rn(x)) : __half_as_ushort(__float2half_rn(x));
}

// One row is handled by D / VEC consecutive lanes of one warp; every lane
// loads the row's two LSE values, the first lane stores the merged one after
// the others have read the old (the running LSE is updated in place).
template <bool BF16, bool HAS_ACC, bool FINAL>
__global__ void __launch_bounds__(THREADS) merge_kernel(const __grid_constant__ Params p) {
  const int per_row = p.D / VEC;                    // 8 or 16 lanes, a divisor of 32
  const long long total = p.rows * per_row;         // a multiple of per_row
  const int lane = threadIdx.x & 31;
  const unsigned row_mask = ((per_row == 32) ? 0xffffffffu : ((1u << per_row) - 1u)) << (lane & ~(per_row - 1));
  const long long stride = (long long)gridDim.x * THREADS;
  for (long long g = (long long)blockIdx.x * THREADS + threadIdx.x; g < total; g += stride) {
    const long long r = g / per_row;
    const int c = (int)(g - r * per_row);
    long long li = r;                               // the row's LSE index, [B, H, S]
    if (!p.bhsd) {                                  // r = (b * S + s) * H + h
      const long long bs = r / p.H;
      const int h = (int)(r - bs * p.H);
      const long long b = bs / p.S;
      const int s = (int)(bs - b * p.S);
      li = (b * p.H + h) * p.S + s;
    }
    const float lp = p.lse_part[li];
    const float la = HAS_ACC ? p.lse_acc[li] : -INFINITY;
    const float m = fmaxf(lp, la);
    float wp = 0.f, wa = 0.f, lse = -INFINITY;
    if (m != -INFINITY) {
      wp = expf(lp - m);
      wa = HAS_ACC ? expf(la - m) : 0.f;
      const float sum = wp + wa;
      lse = m + logf(sum);
      const float inv = 1.f / sum;
      wp *= inv;
      wa *= inv;
    }
    const size_t e0 = (size_t)r * p.D + (size_t)c * VEC;
    const uint4 raw = *reinterpret_cast<const uint4*>(p.o_part + e0);
    const uint16_t* ph = reinterpret_cast<const uint16_t*>(&raw);
    float v[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) v[i] = wp * to_f32(ph[i], BF16);
    if (HAS_ACC) {
      const float4 a0 = *reinterpret_cast<const float4*>(p.o_acc + e0);
      const float4 a1 = *reinterpret_cast<const float4*>(p.o_acc + e0 + 4);
      v[0] = fmaf(wa, a0.x, v[0]); v[1] = fmaf(wa, a0.y, v[1]);
      v[2] = fmaf(wa, a0.z, v[2]); v[3] = fmaf(wa, a0.w, v[3]);
      v[4] = fmaf(wa, a1.x, v[4]); v[5] = fmaf(wa, a1.y, v[5]);
      v[6] = fmaf(wa, a1.z, v[6]); v[7] = fmaf(wa, a1.w, v[7]);
    }
    if (FINAL) {
      uint4 out;
      uint16_t* oh = reinterpret_cast<uint16_t*>(&out);
#pragma unroll
      for (int i = 0; i < VEC; ++i) oh[i] = from_f32(v[i], BF16);
      *reinterpret_cast<uint4*>(p.o_out + e0) = out;
      if (c == 0) p.lse_out[li] = lse;
    } else {
      *reinterpret_cast<float4*>(p.o_acc + e0) = make_float4(v[0], v[1], v[2], v[3]);
      *reinterpret_cast<float4*>(p.o_acc + e0 + 4) = make_float4(v[4], v[5], v[6], v[7]);
      __syncwarp(row_mask);                         // every lane of the row has read lse_acc
      if (c == 0) p.lse_acc[li] = lse;
    }
  }
}

// Split-KV: a row's nsplit partial results, each normalised over its own key
// range (fp32 O at row s * S + r of a [B * H, nsplit * S, D] buffer, its LSE
// at the same row of [B * H, nsplit * S]), merged in one pass by the same
// update taken over all of them at once:
//   LSE = M + log(sum_s exp(LSE_s - M)),  O = sum_s exp(LSE_s - LSE) O_s,
// with M the largest LSE_s (a split with LSE_s = -inf has weight 0).  One warp
// per row, D / 32 columns per lane; O is written in the 16-bit input type in
// the caller's layout, LSE as fp32 [B, H, S].
template <int D, bool BF16>
__global__ void __launch_bounds__(THREADS) splitkv_merge_kernel(const float* __restrict__ o_part,
                                                                const float* __restrict__ lse_part, uint16_t* o,
                                                                float* lse, long long rows, int H, int S, int nsplit,
                                                                int bhsd) {
  constexpr int PER = D / 32;
  constexpr float LOG2E = 1.44269504088896340736f;
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * (THREADS / 32) + (threadIdx.x >> 5);   // [B, H, S] order
  if (row >= rows) return;
  const long long bh = row / S;
  const int r = (int)(row - bh * S);
  const size_t base = (size_t)bh * nsplit * S + r;
  // lane l holds the LSEs of splits l and l + 32 (nsplit <= 64) and their weights
  const float l0 = lane < nsplit ? lse_part[base + (size_t)lane * S] : -INFINITY;
  const float l1 = lane + 32 < nsplit ? lse_part[base + (size_t)(lane + 32) * S] : -INFINITY;
  float m = fmaxf(l0, l1);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  const float e0 = (m > -INFINITY && l0 > -INFINITY) ? ex2((l0 - m) * LOG2E) : 0.f;
  const float e1 = (m > -INFINITY && l1 > -INFINITY) ? ex2((l1 - m) * LOG2E) : 0.f;
  float wsum = e0 + e1;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, off);
  float acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) acc[i] = 0.f;
  // four splits' rows in flight at a time (a split of weight 0 is not read)
  for (int s0 = 0; s0 < nsplit; s0 += 4) {
    float w[4];
    float x[4][PER];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int sp = s0 + u;
      const float e = __shfl_sync(0xffffffffu, sp < 32 ? e0 : e1, sp & 31);
      w[u] = sp < nsplit ? e : 0.f;
      const float* src = o_part + (base + (size_t)sp * S) * D + lane * PER;
      if (w[u] != 0.f) {
        if constexpr (PER == 4) {
          const float4 v = *reinterpret_cast<const float4*>(src);
          x[u][0] = v.x; x[u][1] = v.y; x[u][2] = v.z; x[u][3] = v.w;
        } else {
          const float2 v = *reinterpret_cast<const float2*>(src);
          x[u][0] = v.x; x[u][1] = v.y;
        }
      } else {
#pragma unroll
        for (int i = 0; i < PER; ++i) x[u][i] = 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int i = 0; i < PER; ++i) acc[i] += w[u] * x[u][i];
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  const long long b = bh / H, h = bh - b * H;
  const size_t orow = bhsd ? (size_t)(bh * S + r) : (size_t)((b * S + r) * H + h);
  uint16_t* dst = o + orow * D + lane * PER;
  uint32_t w2[PER / 2];
#pragma unroll
  for (int i = 0; i < PER / 2; ++i)
    w2[i] = (uint32_t)from_f32(acc[2 * i] * inv, BF16) | ((uint32_t)from_f32(acc[2 * i + 1] * inv, BF16) << 16);
  if constexpr (PER == 4) *reinterpret_cast<uint2*>(dst) = make_uint2(w2[0], w2[1]);
  else *reinterpret_cast<uint32_t*>(dst) = w2[0];
  if (lane == 0) lse[row] = m > -INFINITY ? m + lg2(wsum) * 0.69314718055994530942f : -INFINITY;
}

}  // namespace merge
}  // namespace fa

namespace {

template <bool BF16>
fa_status launch_merge(const fa::merge::Params& prm, bool has_acc, bool final_, int grid, cudaStream_t s) {
  using namespace fa::merge;
  if (has_acc && final_) merge_kernel<BF16, true, true><<<grid, THREADS, 0, s>>>(prm);
  else if (has_acc) merge_kernel<BF16, true, false><<<grid, THREADS, 0, s>>>(prm);
  else if (final_) merge_kernel<BF16, false, true><<<grid, THREADS, 0, s>>>(prm);
  else merge_kernel<BF16, false, false><<<grid, THREADS, 0, s>>>(prm);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FA_OK : cuda_fail((int)e);
}

}  // namespace

extern "C" {

fa_status fa_lse_merge(const void* o_part, const float* lse_part, float* o_acc, float* lse_acc, void* o_out,
                       float* lse_out, int64_t B, int64_t H, int64_t S, int64_t D, fa_layout layout,
                       fa_dtype dtype, int flags, void* stream) {
  if (B <= 0 || H <= 0 || S < 0 || D <= 0) return FA_ERR_INVALID_ARG;
  if (layout != FA_BSND && layout != FA_BHSD) return FA_ERR_INVALID_ARG;
  if (dtype != FA_FP16 && dtype != FA_BF16) return FA_ERR_INVALID_ARG;
  if (flags & ~(FA_MERGE_ACCUMULATE | FA_MERGE_FINAL)) return FA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  const int64_t lim = (int64_t)1 << 30;
  if (B >= lim || H >= lim || S >= lim || B * H >= lim) return FA_ERR_UNSUPPORTED;
  if (S == 0) return FA_OK;
  const bool has_acc = (flags & FA_MERGE_ACCUMULATE) != 0, final_ = (flags & FA_MERGE_FINAL) != 0;
  // the running result is read when accumulating and written unless final
  const bool need_acc = has_acc || !final_;
  if (!o_part || !lse_part) return FA_ERR_INVALID_ARG;
  if (need_acc && (!o_acc || !lse_acc)) return FA_ERR_INVALID_ARG;
  if (final_ && (!o_out || !lse_out)) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(o_part) | (need_acc ? reinterpret_cast<uintptr_t>(o_acc) : 0) |
       (final_ ? reinterpret_cast<uintptr_t>(o_out) : 0)) & 15u)
    return FA_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(lse_part) | (need_acc ? reinterpret_cast<uintptr_t>(lse_acc) : 0) |
       (final_ ? reinterpret_cast<uintptr_t>(lse_out) : 0)) & 3u)
    return FA_ERR_MISALIGNED;
  const size_t n = (size_t)(B * H * S);
  const size_t ob = n * (size_t)D * 2, ab = n * (size_t)D * 4, lb = n * 4;
  // outputs may not overlap other arrays (the running result is updated in place)
  if (final_) {
    if (overlaps(o_out, ob, o_part, ob) || overlaps(o_out, ob, lse_part, lb) || overlaps(lse_out, lb, o_part, ob) ||
        overlaps(lse_out, lb, lse_part, lb) || overlaps(o_out, ob, lse_out, lb))
      return FA_ERR_ALIAS;
    if (has_acc && (overlaps(o_out, ob, o_acc, ab) || overlaps(o_out, ob, lse_acc, lb) ||
                    overlaps(lse_out, lb, o_acc, ab) || overlaps(lse_out, lb, lse_acc, lb)))
      return FA_ERR_ALIAS;
  }
  if (need_acc && (overlaps(o_acc, ab, o_part, ob) || overlaps(o_acc, ab, lse_part, lb) ||
                   overlaps(lse_acc, lb, o_part, ob) || overlaps(lse_acc, lb, lse_part, lb) ||
                   overlaps(o_acc, ab, lse_acc, lb)))
    return FA_ERR_ALIAS;

  int dev = 0, sms = 0;
  const void* ptrs[6] = {o_part, lse_part, need_acc ? o_acc : nullptr, need_acc ? lse_acc : nullptr,
                         final_ ? o_out : nullptr, final_ ? lse_out : nullptr};
  fa_status st = device_checks(ptrs, 6, &dev, &sms);
  if (st != FA_OK) return st;

  fa::merge::Params prm;
  prm.o_part = static_cast<const uint16_t*>(o_part);
  prm.lse_part = lse_part;
  prm.o_acc = o_acc;
  prm.lse_acc = lse_acc;
  prm.o_out = static_cast<uint16_t*>(o_out);
  prm.lse_out = lse_out;
  prm.rows = (long long)n;
  prm.H = (int)H;
  prm.S = (int)S;
  prm.D = (int)D;
  prm.bhsd = layout == FA_BHSD ? 1 : 0;
  // a memory-bound pass: enough resident threads to cover HBM latency, grid-stride beyond
  const long long threads = (long long)n * (D / fa::merge::VEC);
  const long long want = (threads + fa::merge::THREADS - 1) / fa::merge::THREADS;
  const long long cap = (long long)sms * 8;
  const int grid = (int)(want < cap ? want : cap);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return dtype == FA_BF16 ? launch_merge<true>(prm, has_acc, final_, grid, s)
                          : launch_merge<false>(prm, has_acc, final_, grid, s);
}

// Workspace of fa_fwd_splitkv: the work counter (256 bytes kept for it), the
// partial LSEs and the partial O rows, all for nsplit splits.
static size_t splitkv_ws_bytes(int64_t B, int64_t H, int64_t Sq, int64_t D, int64_t nsplit) {
  const size_t rows = (size_t)(B * H * nsplit * Sq);
  return 256 + ((rows * 4 + 15) & ~(size_t)15) + rows * (size_t)D * 4;
}

size_t fa_fwd_splitkv_workspace_size(int64_t B, int64_t H, int64_t Sq, int64_t D, int nsplit) {
  if (B <= 0 || H <= 0 || Sq < 0 || (D != 64 && D != 128) || nsplit < 1 || nsplit > 64) return 0;
  return splitkv_ws_bytes(B, H, Sq, D, nsplit);
}

fa_status fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t H,
                         int64_t Sq, int64_t Sk, int64_t D, fa_layout layout, float scale, fa_dtype dtype, int nsplit,
                         void* workspace, size_t workspace_bytes, void* stream) {
  bool noop = false;
  fa_status hst = host_checks(q, k, v, o, lse, B, H, Sq, Sk, D, layout, scale, dtype, &noop);
  if (hst != FA_OK) return hst;
  if (nsplit < 1 || nsplit > 64) return FA_ERR_INVALID_ARG;
  if (noop) return FA_OK;
  // splits of whole key tiles: split_keys keys each (the last may be shorter)
  const int64_t per = (Sk + nsplit - 1) / nsplit;
  const int64_t split_keys = (per + fa::BN - 1) / fa::BN * fa::BN;
  const int64_t n_eff = (Sk + split_keys - 1) / split_keys;
  const size_t need = splitkv_ws_bytes(B, H, Sq, D, n_eff);
  if (!workspace || workspace_bytes < splitkv_ws_bytes(B, H, Sq, D, nsplit) || workspace_bytes < need)
    return FA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return FA_ERR_MISALIGNED;
  const int64_t nqb = (Sq + fa::UNIT_ROWS - 1) / fa::UNIT_ROWS;
  if (n_eff * B * H * nqb >= ((int64_t)1 << 30) || B * H * n_eff * Sq >= ((int64_t)1 << 31)) return FA_ERR_UNSUPPORTED;
  {
    const size_t qbytes = (size_t)(B * H * Sq * D) * 2, kvbytes = (size_t)(B * H * Sk * D) * 2;
    const size_t lbytes = (size_t)(B * H * Sq) * 4;
    const void* bufs[5] = {q, k, v, o, lse};
    const size_t sizes[5] = {qbytes, kvbytes, kvbytes, qbytes, lbytes};
    for (int j = 0; j < 5; ++j)
      if (overlaps(workspace, workspace_bytes, bufs[j], sizes[j])) return FA_ERR_ALIAS;
  }
  int dev = 0, sms = 0;
  const void* ptrs[6] = {q, k, v, o, lse, workspace};
  fa_status st = device_checks(ptrs, 6, &dev, &sms);
  if (st != FA_OK) return st;
  CUtensorMap mq, mk, mv;
  if ((st = make_map(&mq, q, dtype, layout, B, H, Sq, D)) != FA_OK) return st;
  if ((st = make_map(&mk, k, dtype, layout, B, H, Sk, D)) != FA_OK) return st;
  if ((st = make_map(&mv, v, dtype, layout, B, H, Sk, D)) != FA_OK) return st;

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* lse_part = reinterpret_cast<float*>(ws + 256);
  const size_t prow = (size_t)(B * H * n_eff * Sq);
  float* o_part = reinterpret_cast<float*>(ws + 256 + ((prow * 4 + 15) & ~(size_t)15));

  fa::Params prm{};
  prm.lse = lse_part;
  prm.acc = o_part;
  prm.o = static_cast<uint8_t*>(o);        // not written: every split's result is a partial
  prm.o_bs = H * n_eff * Sq * D;
  prm.o_hs = n_eff * Sq * D;
  prm.o_rs = D;
  prm.lse_bs = H * n_eff * Sq;
  prm.lse_hs = n_eff * Sq;
  prm.B = (int)B;
  prm.H = (int)H;
  prm.Sq = (int)Sq;
  prm.Sk = (int)Sk;
  prm.nqb = (int)nqb;
  prm.tk = (int)((split_keys + fa::BN - 1) / fa::BN);
  prm.bh = (int)(B * H);
  prm.head0 = 0;
  prm.group_heads = l2_group_heads(split_keys, D, B * H);
  prm.total_units = (int)(n_eff * B * H * nqb);
  prm.causal = 0;
  prm.bhsd = layout == FA_BHSD ? 1 : 0;
  prm.scale_log2 = (float)((double)scale * 1.4426950408889634074);
  prm.wait_limit_ns = 1000000000ull;
  prm.withhold_loads = 0;
  set_softmax_params(prm, SoftmaxOpts());
  prm.nseg = 1;                 // the ring-step kind, in its split mode
  prm.seg_units0 = (int)(B * H * nqb);
  prm.split_n = (int)n_eff;
  prm.split_keys = (int)split_keys;
  st = launch_units(prm, mq, mk, mv, mq, D, dtype, reinterpret_cast<unsigned int*>(ws), dev, sms, stream);
  if (st != FA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const long long rows = B * H * Sq;
  const unsigned grid = (unsigned)((rows + fa::merge::THREADS / 32 - 1) / (fa::merge::THREADS / 32));
  uint16_t* o16 = static_cast<uint16_t*>(o);
  const int bhsd = layout == FA_BHSD ? 1 : 0;
  if (D == 128) {
    if (dtype == FA_BF16)
      fa::merge::splitkv_merge_kernel<128, true><<<grid, fa::merge::THREADS, 0, s>>>(o_part, lse_part, o16, lse, rows, (int)H, (int)Sq, (int)n_eff, bhsd);
    else
      fa::merge::splitkv_merge_kernel<128, false><<<grid, fa::merge::THREADS, 0, s>>>(o_part, lse_part, o16, lse, rows, (int)H, (int)Sq, (int)n_eff, bhsd);
  } else {
    if (dtype == FA_BF16)
      fa::merge::splitkv_merge_kernel<64, true><<<grid, fa::merge::THREADS, 0, s>>>(o_part, lse_part, o16, lse, rows, (int)H, (int)Sq, (int)n_eff, bhsd);
    else
      fa::merge::splitkv_merge_kernel<64, false><<<grid, fa::merge::THREADS, 0, s>>>(o_part, lse_part, o16, lse, rows, (int)H, (int)Sq, (int)n_eff, bhsd);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail((int)e);
  return FA_OK;
}

}  // extern "C"
