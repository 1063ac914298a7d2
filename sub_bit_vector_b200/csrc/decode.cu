// Fused split-K decode attention from loop-axis VQ codes (sm_100a).
//
// LoopVQ project page, "Serving in SGLang -- Attend from indices": at loop
// step t the kernel reads keys and values from the shared index rows through
// the step's codebook slice B_t and merges them with the bf16 sink/recent
// attention.  One CTA handles one split of one (request, query head):
//
//   window split : the bf16 sink + recent tokens, online softmax in fp32.
//   body split   : up to kSplitCap tokens of codes, in two passes over a
//                  TMA-fed shared-memory ring:
//     pass K  -- score s_n = sum_j LUT[j][idxK[n][j]] with the per-step
//                lookup table LUT[j][c] = scale*log2(e) * q_j . B^K_t[c][j];
//                lane l owns slot l%J, so a warp-wide gather touches 32
//                distinct banks; the J partial sums of a token are added by
//                a select-free butterfly (the K tile byte order puts token
//                i^j in register i of lane j).
//     pass V  -- with the split maximum m known, token weight
//                p_n = 2^(s_n - m) in (0, 1] becomes a u32 fixed-point
//                q_n = floor(p_n 2^S + u_n) (u_n a Weyl dither, so the
//                rounding is unbiased) and is added into a per-slot 256-bin
//                histogram hist[j][idxV[n][j]] with shared-memory integer
//                atomics (one bank per lane, conflict free);
//     epilogue   -- o[jW+w] = 2^-S sum_c hist[j][c] B^V_t[c][j][w].
//   The last CTA of a (request, head) merges the splits' (m, l, o) by
//   log-sum-exp (atomic ticket, no waiting).
//
// Fixed-point bound: a split holds n <= kSplitCap < 2^12 tokens and S is
// chosen so that n * 2^S < 2^32, so no bin or sum can overflow.

#include <math.h>
#include <stdio.h>

#include "common.cuh"

namespace loopvq {

constexpr int kNW = 16;                      // consumer warps
constexpr int kThreads = (kNW + 1) * 32;     // + one producer warp
constexpr int kStages = 4;
constexpr int kStageBytes = 16384;
constexpr int kSplitCap = 4064;              // max body tokens per split, multiple of 32
constexpr int kRegionAlign = 32768;          // LUT / histogram base alignment
// dynamic smem: alignment pad + LUT (32 KB) + histogram (32 KB) + ring + scores + misc
constexpr int kScoresBytes = kSplitCap * 4;
constexpr int kMiscBytes = 4096;
constexpr int kDynSmem = kRegionAlign + 32768 + 32768 + kStages * kStageBytes + kScoresBytes + kMiscBytes;

struct DecodeParams {
  int T, Tc, H, Hq, D, J, W, C;
  int loop_step;
  float scale_log2;
  int batch, n_sink, n_recent, page, max_ctx;
  const int32_t* ctx_len;
  const int64_t* body_off;
  const int64_t* win_off;
  int64_t body_pool_tokens, win_pool_tokens;
  const void* cbK_slice;   // [H][C][J][W] of step t
  const void* cbV_slice;
  const uint8_t* idxK;     // pool streams of code block t / Tc: [H][pool_tiles][tile]
  const uint8_t* idxV;
  const __nv_bfloat16* winK;  // [H][win_pool][D] of step t
  const __nv_bfloat16* winV;
  const void* q;
  int q_bf16;
  void* out;
  int out_bf16;
  float* lse;
  uint32_t* status;
  uint32_t* tickets;
  float* partials;
  int split_len;   // body tokens per split (multiple of 32, <= kSplitCap)
  int max_splits;  // grid.x
};

__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kNW * 32) : "memory");
}

// Shared address of the LUT / histogram entry of `code` (byte K of w) for
// this lane: rows of 32 words, column = lane.  base is 32 KB aligned, so the
// row offset can be OR-ed in.
template <int K>
__device__ __forceinline__ uint32_t code_addr(uint32_t w, uint32_t base) {
  uint32_t x = (K == 0) ? (w << 7) : (w >> (8 * K - 7));
  return (x & 0x7F80u) | base;
}
__device__ __forceinline__ float lds_f32(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ void red_add_u32(uint32_t a, uint32_t v) {
  asm volatile("red.shared.add.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}

template <int J>
__device__ __forceinline__ void load_lane_words(const uint8_t* p, uint32_t (&w)[J / 4]) {
  if constexpr (J == 32) {
    uint4 a = *reinterpret_cast<const uint4*>(p);
    uint4 b = *reinterpret_cast<const uint4*>(p + 16);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
  } else if constexpr (J == 16) {
    uint4 a = *reinterpret_cast<const uint4*>(p);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
  } else {
    uint2 a = *reinterpret_cast<const uint2*>(p);
    w[0] = a.x; w[1] = a.y;
  }
}

// Score of token `lane` of a K tile (lane's J bytes at p).
template <int J>
__device__ __forceinline__ float tile_scores(const uint8_t* p, uint32_t lut_lane) {
  uint32_t w[J / 4];
  load_lane_words<J>(p, w);
  float v[J];
#pragma unroll
  for (int i = 0; i < J / 4; ++i) {
    v[4 * i + 0] = lds_f32(code_addr<0>(w[i], lut_lane));
    v[4 * i + 1] = lds_f32(code_addr<1>(w[i], lut_lane));
    v[4 * i + 2] = lds_f32(code_addr<2>(w[i], lut_lane));
    v[4 * i + 3] = lds_f32(code_addr<3>(w[i], lut_lane));
  }
#pragma unroll
  for (int m = J / 2; m >= 1; m >>= 1) {
#pragma unroll
    for (int i = 0; i < m; ++i) v[i] += __shfl_xor_sync(0xffffffffu, v[i + m], m);
  }
  return v[0];
}

// Adds the weights of the group's J tokens into the histogram columns of this
// lane for one V tile (lane's J bytes at p; weights at qg[0..J)).
template <int J>
__device__ __forceinline__ void tile_hist(const uint8_t* p, const uint32_t* qg, uint32_t hist_lane) {
  uint32_t w[J / 4];
  load_lane_words<J>(p, w);
#pragma unroll
  for (int i = 0; i < J / 4; ++i) {
    uint4 qq = *reinterpret_cast<const uint4*>(qg + 4 * i);
    red_add_u32(code_addr<0>(w[i], hist_lane), qq.x);
    red_add_u32(code_addr<1>(w[i], hist_lane), qq.y);
    red_add_u32(code_addr<2>(w[i], hist_lane), qq.z);
    red_add_u32(code_addr<3>(w[i], hist_lane), qq.w);
  }
}

// Loads W consecutive codebook elements (bf16 or fp32) as fp32; zero if !ok.
template <int W, typename CBT>
__device__ __forceinline__ void load_vec(const CBT* p, bool ok, float (&v)[W]) {
  if constexpr (sizeof(CBT) == 2) {
    static_assert(W % 4 == 0 || W == 2, "bf16 vectors of 2, 4, 8 or 16");
    if constexpr (W == 2) {
      const uint32_t a = ok ? *reinterpret_cast<const uint32_t*>(p) : 0u;
      v[0] = bf16_lo(a); v[1] = bf16_hi(a);
    } else {
#pragma unroll
      for (int i = 0; i < W; i += 4) {
        const uint2 a = ok ? *reinterpret_cast<const uint2*>(p + i) : make_uint2(0u, 0u);
        v[i] = bf16_lo(a.x); v[i + 1] = bf16_hi(a.x); v[i + 2] = bf16_lo(a.y); v[i + 3] = bf16_hi(a.y);
      }
    }
  } else {
    if constexpr (W == 2) {
      const float2 a = ok ? *reinterpret_cast<const float2*>(p) : make_float2(0.f, 0.f);
      v[0] = a.x; v[1] = a.y;
    } else {
#pragma unroll
      for (int i = 0; i < W; i += 4) {
        const float4 a = ok ? *reinterpret_cast<const float4*>(p + i) : make_float4(0.f, 0.f, 0.f, 0.f);
        v[i] = a.x; v[i + 1] = a.y; v[i + 2] = a.z; v[i + 3] = a.w;
      }
    }
  }
}

__device__ __forceinline__ float load_q(const void* q, int q_bf16, size_t i) {
  return q_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(q)[i])
                : reinterpret_cast<const float*>(q)[i];
}

template <int J, int D, typename CBT>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const DecodeParams p) {
  extern __shared__ __align__(1024) uint8_t dyn[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, hq = blockIdx.y, r = blockIdx.z;
  const int group = p.Hq / p.H;
  const int h = hq / group;
  constexpr int W = D / J;

  // ---- work of this CTA -------------------------------------------------
  int ctx = __ldg(p.ctx_len + r);
  bool bad = false;
  if (ctx < 0 || ctx > p.max_ctx) {
    if (tid == 0 && split == 0) set_fault(p.status, LOOPVQ_FAULT_CTX_RANGE);
    ctx = 0;
  }
  const CtxSplit cs = ctx_split(ctx, p.n_sink, p.n_recent, p.page);
  const int n_win = cs.sink + cs.recent;
  const int has_win = n_win > 0 ? 1 : 0;
  const int n_body_splits = (cs.body + p.split_len - 1) / p.split_len;
  const int n_splits = has_win + n_body_splits;
  const size_t unit = (size_t)r * p.Hq + hq;
  if (ctx == 0) {  // empty context: zero output, lse -inf
    if (split == 0) {
      for (int d = tid; d < D; d += blockDim.x) {
        if (p.out_bf16) reinterpret_cast<__nv_bfloat16*>(p.out)[unit * D + d] = __float2bfloat16_rn(0.f);
        else reinterpret_cast<float*>(p.out)[unit * D + d] = 0.f;
      }
      if (p.lse && tid == 0) p.lse[unit] = -INFINITY;
    }
    return;
  }
  if (split >= n_splits) return;
  const bool is_window = split < has_win;
  const int bsplit = split - has_win;
  int64_t win_off = 0, body_off = 0;
  if (is_window) {
    win_off = __ldg(p.win_off + r);
    if (win_off < 0 || win_off + n_win > p.win_pool_tokens) bad = true;
  } else {
    body_off = __ldg(p.body_off + r);
    if (body_off < 0 || (body_off & 31) || body_off + cs.body > p.body_pool_tokens) bad = true;
  }
  if (bad && tid == 0) set_fault(p.status, LOOPVQ_FAULT_POOL_RANGE);
  const int tok0 = is_window ? 0 : bsplit * p.split_len;
  const int n_tok = bad ? 0 : (is_window ? n_win : min(p.split_len, cs.body - tok0));
  const int n_tiles = (n_tok + 31) >> 5;

  // ---- shared memory plan ------------------------------------------------
  const uint32_t sbase = smem_u32(dyn);
  const uint32_t region = (sbase + (kRegionAlign - 1)) & ~(uint32_t)(kRegionAlign - 1);
  uint8_t* const dyn_region = dyn + (region - sbase);
  float* const lut = reinterpret_cast<float*>(dyn_region);                 // [256][32]
  uint32_t* const hist = reinterpret_cast<uint32_t*>(dyn_region + 32768);  // [256][32]
  uint8_t* const ring = dyn_region + 65536;
  float* const sc = reinterpret_cast<float*>(ring + kStages * kStageBytes);
  uint8_t* const misc = reinterpret_cast<uint8_t*>(sc) + kScoresBytes;
  uint64_t* const full_bar = reinterpret_cast<uint64_t*>(misc);
  uint64_t* const empty_bar = full_bar + kStages;
  float* const qs = reinterpret_cast<float*>(misc + 128);         // [D <= 128] scaled query
  float* const red = reinterpret_cast<float*>(misc + 128 + 512);  // [kNW * 2]
  uint32_t* const qbuf = reinterpret_cast<uint32_t*>(misc + 1024);  // [kNW][32]
  int* const flag = reinterpret_cast<int*>(misc + 1024 + kNW * 128);

  // chunks: window -> one chunk per 32 tokens (K rows then V rows);
  //         body   -> K tiles then V tiles, tiles_per_chunk each.
  constexpr int kTilesPerChunk = kStageBytes / (32 * J);
  const int n_chunks_half = is_window ? (n_tok + 31) / 32 : (n_tiles + kTilesPerChunk - 1) / kTilesPerChunk;
  const int n_chunks = is_window ? n_chunks_half : 2 * n_chunks_half;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(full_bar + s), 1);
      mbar_init(smem_u32(empty_bar + s), kNW);
    }
    fence_mbar_init();
  }
  __syncthreads();

  // ======================= producer warp ===================================
  if (warp == kNW) {
    if (lane == 0) {
      for (int k = 0; k < n_chunks; ++k) {
        const int s = k % kStages;
        if (k >= kStages) {
          if (!mbar_wait_bounded(smem_u32(empty_bar + s), ((k / kStages) - 1) & 1)) {
            set_fault(p.status, LOOPVQ_FAULT_TIMEOUT);
            break;
          }
        }
        const uint32_t dst = smem_u32(ring + s * kStageBytes);
        const uint32_t fb = smem_u32(full_bar + s);
        if (is_window) {
          const int t0 = k * 32;
          const int nt = min(32, n_tok - t0);
          const uint32_t bytes = (uint32_t)nt * D * 2;
          const size_t row0 = ((size_t)h * p.win_pool_tokens + win_off + t0) * D;
          mbar_arrive_expect_tx(fb, 2 * bytes);
          bulk_g2s(dst, p.winK + row0, bytes, fb);
          bulk_g2s(dst + 32 * D * 2, p.winV + row0, bytes, fb);
        } else {
          const bool vpass = k >= n_chunks_half;
          const int c = vpass ? k - n_chunks_half : k;
          const int tl0 = c * kTilesPerChunk;
          const int nt = min(kTilesPerChunk, n_tiles - tl0);
          const uint32_t bytes = (uint32_t)nt * 32 * J;
          const int64_t tile = ((body_off + tok0) >> 5) + tl0;
          const uint8_t* src = (vpass ? p.idxV : p.idxK) + ((int64_t)h * (p.body_pool_tokens >> 5) + tile) * (32 * J);
          mbar_arrive_expect_tx(fb, bytes);
          bulk_g2s(dst, src, bytes, fb);
        }
      }
    }
    return;
  }

  // ======================= consumer warps ==================================
  float* const part = p.partials + (unit * p.max_splits + split) * (size_t)(D + 4);
  const int ctid = tid;  // 0 .. kNW*32-1

  // scaled query (log2 units)
  for (int d = ctid; d < D; d += kNW * 32) qs[d] = load_q(p.q, p.q_bf16, unit * D + d) * p.scale_log2;
  consumer_sync();

  if (is_window) {
    // lane owns channels lane*CPL .. lane*CPL+CPL-1 (CPL = D/32 = 2 or 4)
    constexpr int CPL = D >> 5;
    float qv[4], ov[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < CPL; ++i) qv[i] = qs[lane * CPL + i];
    float m = -INFINITY, l = 0.f;
    for (int k = 0; k < n_chunks; ++k) {
      const int s = k % kStages;
      if (!mbar_wait_bounded(smem_u32(full_bar + s), (k / kStages) & 1)) set_fault(p.status, LOOPVQ_FAULT_TIMEOUT);
      const uint8_t* st = ring + s * kStageBytes;
      const int nt = min(32, n_tok - k * 32);
      for (int tkn = warp; tkn < nt; tkn += kNW) {
        const uint8_t* kr = st + (size_t)tkn * D * 2 + lane * CPL * 2;
        const uint8_t* vr = st + 32 * D * 2 + (size_t)tkn * D * 2 + lane * CPL * 2;
        float kf[4], vf[4];
        if constexpr (CPL == 4) {
          uint2 a = *reinterpret_cast<const uint2*>(kr);
          uint2 b = *reinterpret_cast<const uint2*>(vr);
          kf[0] = bf16_lo(a.x); kf[1] = bf16_hi(a.x); kf[2] = bf16_lo(a.y); kf[3] = bf16_hi(a.y);
          vf[0] = bf16_lo(b.x); vf[1] = bf16_hi(b.x); vf[2] = bf16_lo(b.y); vf[3] = bf16_hi(b.y);
        } else {
          uint32_t a = *reinterpret_cast<const uint32_t*>(kr);
          uint32_t b = *reinterpret_cast<const uint32_t*>(vr);
          kf[0] = bf16_lo(a); kf[1] = bf16_hi(a); kf[2] = kf[3] = 0.f;
          vf[0] = bf16_lo(b); vf[1] = bf16_hi(b); vf[2] = vf[3] = 0.f;
        }
        float sdot = 0.f;
#pragma unroll
        for (int i = 0; i < CPL; ++i) sdot = fmaf(qv[i], kf[i], sdot);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) sdot += __shfl_xor_sync(0xffffffffu, sdot, o);
        if (sdot > m) {
          const float corr = exp2f(m - sdot);
          l *= corr;
#pragma unroll
          for (int i = 0; i < 4; ++i) ov[i] *= corr;
          m = sdot;
        }
        const float pw = exp2f(sdot - m);
        l += pw;
#pragma unroll
        for (int i = 0; i < CPL; ++i) ov[i] = fmaf(pw, vf[i], ov[i]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(empty_bar + s));
    }
    // merge the warps' (m, l, o): reuse the score buffer as [kNW][D + 2]
    float* wpart = sc;
#pragma unroll
    for (int i = 0; i < CPL; ++i) wpart[warp * (D + 2) + lane * CPL + i] = ov[i];
    if (lane == 0) {
      wpart[warp * (D + 2) + D] = m;
      wpart[warp * (D + 2) + D + 1] = l;
    }
    consumer_sync();
    float M = -INFINITY;
    for (int w = 0; w < kNW; ++w) M = fmaxf(M, wpart[w * (D + 2) + D]);
    for (int d = ctid; d < D + 2; d += kNW * 32) {
      float acc = 0.f;
      if (d < D || d == D + 1) {
        for (int w = 0; w < kNW; ++w) {
          const float mw = wpart[w * (D + 2) + D];
          if (mw != -INFINITY) acc += wpart[w * (D + 2) + d] * exp2f(mw - M);
        }
      }
      part[d] = (d == D) ? M : acc;
    }
  } else {
    // ---- LUT of step t: LUT[c][g*J + j] = sum_w qs[j*W+w] * B^K_t[c][j][w].
    // Entry e = (c, j) is one W-vector of the code-major slice; a thread owns
    // entries ctid + 512k, all loads issued before any use.
    const CBT* bk = reinterpret_cast<const CBT*>(p.cbK_slice) + (size_t)h * p.C * J * W;
    {
      constexpr int kPer = 256 * J / (kNW * 32);
      float wv[kPer][W];
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const int e = ctid + k * kNW * 32;
        const int c = e / J;
        load_vec<W>(bk + (size_t)e * W, c < p.C, wv[k]);
      }
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const int e = ctid + k * kNW * 32;
        const int c = e / J, j = e % J;
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < W; ++w) acc = fmaf(qs[j * W + w], wv[k][w], acc);
        if (c >= p.C) acc = __int_as_float(0x7fc00000);  // NaN marks a code >= n_codes
#pragma unroll
        for (int g = 0; g < 32 / J; ++g) lut[c * 32 + g * J + j] = acc;
      }
    }
    for (int e = ctid; e < 256 * 32; e += kNW * 32) hist[e] = 0u;
    consumer_sync();

    const uint32_t lut_lane = region + lane * 4;
    const uint32_t hist_lane = region + 32768 + lane * 4;
    // ---- pass K: scores and split maximum
    float mx = -INFINITY;
    bool nan_seen = false;
    for (int k = 0; k < n_chunks_half; ++k) {
      const int s = k % kStages;
      if (!mbar_wait_bounded(smem_u32(full_bar + s), (k / kStages) & 1)) set_fault(p.status, LOOPVQ_FAULT_TIMEOUT);
      const uint8_t* st = ring + s * kStageBytes;
      const int nt = min(kTilesPerChunk, n_tiles - k * kTilesPerChunk);
      for (int tl = warp; tl < nt; tl += kNW) {
        const float sv = tile_scores<J>(st + tl * 32 * J + lane * J, lut_lane);
        const int tok = (k * kTilesPerChunk + tl) * 32 + lane;
        const bool valid = tok < n_tok;
        if (valid && sv != sv) nan_seen = true;
        const float s2 = valid ? sv : -INFINITY;
        sc[tok] = s2;
        mx = fmaxf(mx, s2);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(empty_bar + s));
    }
    if (nan_seen) set_fault(p.status, LOOPVQ_FAULT_CODE_RANGE);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) red[warp] = mx;
    consumer_sync();
    float m = -INFINITY;
    for (int w = 0; w < kNW; ++w) m = fmaxf(m, red[w]);
    // fixed-point scale: n_tok * 2^S < 2^32
    const int S = 31 - (31 - __clz(max(n_tok, 1)));
    const float scaleS = exp2f((float)S);

    // ---- pass V: weights into the histogram
    uint32_t qsum = 0;
    uint32_t* const qw = qbuf + warp * 32;
    const int g0 = (lane / J) * J;
    for (int k = n_chunks_half; k < n_chunks; ++k) {
      const int s = k % kStages;
      if (!mbar_wait_bounded(smem_u32(full_bar + s), (k / kStages) & 1)) set_fault(p.status, LOOPVQ_FAULT_TIMEOUT);
      const uint8_t* st = ring + s * kStageBytes;
      const int kv = k - n_chunks_half;
      const int nt = min(kTilesPerChunk, n_tiles - kv * kTilesPerChunk);
      for (int tl = warp; tl < nt; tl += kNW) {
        const int tok = (kv * kTilesPerChunk + tl) * 32 + lane;
        uint32_t qv = 0;
        if (tok < n_tok) {
          const float pw = exp2f(sc[tok] - m);
          const uint32_t seq = (uint32_t)(body_off + tok0 + tok);
          const float u = (float)((seq * 2654435769u) >> 8) * (1.0f / 16777216.0f);
          qv = __float2uint_rd(fmaf(pw, scaleS, u));
        }
        qsum += qv;
        qw[lane] = qv;
        __syncwarp();
        tile_hist<J>(st + tl * 32 * J + lane * J, qw + g0, hist_lane);
        __syncwarp();
      }
      if (lane == 0) mbar_arrive(smem_u32(empty_bar + s));
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) qsum += __shfl_xor_sync(0xffffffffu, qsum, o);
    if (lane == 0) reinterpret_cast<uint32_t*>(red)[kNW + warp] = qsum;
    consumer_sync();

    // ---- epilogue: o[d] = 2^-S sum_c hist[j][c] B^V_t[c][j][w].  Thread
    // ctid owns entries e = (c, j) = ctid + 512k and accumulates its W
    // outputs over them; the 512/J partial groups per output are summed
    // through shared memory (the LUT region is free by now).
    const CBT* bv = reinterpret_cast<const CBT*>(p.cbV_slice) + (size_t)h * p.C * D;
    {
      constexpr int kPer = 256 * J / (kNW * 32);
      constexpr int kGroups = (kNW * 32) / J;
      float vv[kPer][W];
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const int e = ctid + k * kNW * 32;
        load_vec<W>(bv + (size_t)e * W, e / J < p.C, vv[k]);
      }
      float acc[W];
#pragma unroll
      for (int w = 0; w < W; ++w) acc[w] = 0.f;
      const int j = ctid % J;
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const int c = (ctid + k * kNW * 32) / J;
        uint32_t hs = 0;
#pragma unroll
        for (int g = 0; g < 32 / J; ++g) hs += hist[c * 32 + g * J + j];
        if (c < p.C) {
          const float hf = (float)hs;
#pragma unroll
          for (int w = 0; w < W; ++w) acc[w] = fmaf(hf, vv[k][w], acc[w]);
        }
      }
      // bins of codes >= n_codes must be empty
      if (p.C < 256) {
        bool any = false;
        for (int e = p.C * 32 + ctid; e < 256 * 32; e += kNW * 32) any |= hist[e] != 0u;
        if (any) set_fault(p.status, LOOPVQ_FAULT_CODE_RANGE);
      }
      float* ored = lut;  // [kGroups][D]
      const int grp = ctid / J;
#pragma unroll
      for (int w = 0; w < W; ++w) ored[grp * D + j * W + w] = acc[w];
      consumer_sync();
      if (ctid < D) {
        float o = 0.f;
#pragma unroll 8
        for (int i = 0; i < kGroups; ++i) o += ored[i * D + ctid];
        part[ctid] = o / scaleS;
      }
    }
    if (ctid == 0) {
      uint64_t tot = 0;
      for (int w = 0; w < kNW; ++w) tot += reinterpret_cast<uint32_t*>(red)[kNW + w];
      part[D] = m;
      part[D + 1] = (float)tot / scaleS;
    }
  }

  // ---- split ticket and combine -------------------------------------------
  __threadfence();
  consumer_sync();
  if (ctid == 0) {
    const uint32_t t = atomicAdd(p.tickets + unit, 1u);
    *flag = (t == (uint32_t)(n_splits - 1)) ? 1 : 0;
  }
  consumer_sync();
  if (*flag) {
    __threadfence();
    combine_splits(p.partials + unit * p.max_splits * (size_t)(D + 4), n_splits, D,
                   p.out_bf16 ? (void*)(reinterpret_cast<__nv_bfloat16*>(p.out) + unit * D)
                              : (void*)(reinterpret_cast<float*>(p.out) + unit * D),
                   p.out_bf16, p.lse ? p.lse + unit : nullptr);
    if (ctid == 0) atomicExch(p.tickets + unit, 0u);
  }
}

// Host-side plan: body tokens per split so that the grid fills the SMs.
struct DecodePlan {
  int n_body_splits, split_len, max_splits;
};
inline DecodePlan decode_plan(int64_t units, int max_body, int n_sm) {
  DecodePlan pl;
  int need = (max_body + kSplitCap - 1) / kSplitCap;  // fixed-point bound
  int fill = (int)(n_sm / (units > 0 ? units : 1)) - 1;  // one window split per unit
  int cap_by_tiles = (max_body + 255) / 256;             // >= 256 tokens per split
  int s = need;
  if (fill > s) s = fill < cap_by_tiles ? fill : cap_by_tiles;
  if (s < 1) s = 1;
  int len = (max_body + s - 1) / s;
  len = ((len + 31) / 32) * 32;
  if (len < 32) len = 32;
  if (len > kSplitCap) len = kSplitCap;
  pl.split_len = len;
  pl.n_body_splits = max_body > 0 ? (max_body + len - 1) / len : 0;
  pl.max_splits = pl.n_body_splits + 1;
  return pl;
}

static int max_body_tokens(const loopvq_cache_layout* L) {
  return ctx_split(L->max_ctx_len, L->n_sink, L->n_recent, L->page).body;
}

// workspace bound independent of the device: plan with a generous SM count
static WsLayout decode_ws(const Geo& g, const loopvq_cache_layout* L) {
  const int64_t units = (int64_t)L->batch * g.Hq;
  DecodePlan pl = decode_plan(units, max_body_tokens(L), 1024);
  return ws_layout(units, pl.max_splits, g.D);
}

static loopvq_status check_layout(const loopvq_cache_layout* L) {
  if (!L || L->batch < 1 || L->n_sink < 0 || L->n_recent < 0 || L->page < 1 || L->max_ctx_len < 0)
    return LOOPVQ_ERR_INVALID_ARG;
  if (!L->ctx_len || !L->body_off || !L->win_off) return LOOPVQ_ERR_INVALID_ARG;
  if (L->body_pool_tokens < 0 || (L->body_pool_tokens & 31) || L->win_pool_tokens < 0) return LOOPVQ_ERR_INVALID_ARG;
  return LOOPVQ_OK;
}

}  // namespace loopvq

using namespace loopvq;

extern "C" size_t loopvq_decode_workspace_bytes(const loopvq_codebook_desc* desc,
                                                const loopvq_cache_layout* layout) {
  Geo g;
  if (make_geo(desc, &g) != LOOPVQ_OK || check_layout(layout) != LOOPVQ_OK) return 0;
  return decode_ws(g, layout).total;
}

extern "C" loopvq_status loopvq_decode_attn(const loopvq_codebook_desc* desc, const void* cbK_packed,
                                            const void* cbV_packed, const loopvq_cache_layout* layout,
                                            const uint8_t* idxK_pool, const uint8_t* idxV_pool,
                                            const void* winK, const void* winV, const void* q,
                                            loopvq_dtype q_dtype, int32_t loop_step, float softmax_scale,
                                            void* out, loopvq_dtype out_dtype, float* lse_out,
                                            void* workspace, size_t workspace_bytes,
                                            loopvq_stream_t stream) {
  Geo g;
  loopvq_status st = make_geo(desc, &g);
  if (st != LOOPVQ_OK) return st;
  if ((st = check_layout(layout)) != LOOPVQ_OK) return st;
  if (g.J != 8 && g.J != 16 && g.J != 32) return LOOPVQ_ERR_UNSUPPORTED;
  if (g.D != 64 && g.D != 128) return LOOPVQ_ERR_UNSUPPORTED;
  if (loop_step < 0 || loop_step >= g.T) return LOOPVQ_ERR_INVALID_ARG;
  if (q_dtype != LOOPVQ_F32 && q_dtype != LOOPVQ_BF16) return LOOPVQ_ERR_INVALID_ARG;
  if (out_dtype != LOOPVQ_F32 && out_dtype != LOOPVQ_BF16) return LOOPVQ_ERR_INVALID_ARG;
  if (!(softmax_scale == softmax_scale)) return LOOPVQ_ERR_INVALID_ARG;
  if (!cbK_packed || !cbV_packed || !idxK_pool || !idxV_pool || !winK || !winV || !q || !out || !workspace)
    return LOOPVQ_ERR_INVALID_ARG;
  if (((uintptr_t)idxK_pool & 15) || ((uintptr_t)idxV_pool & 15) || ((uintptr_t)winK & 15) ||
      ((uintptr_t)winV & 15) || ((uintptr_t)workspace & 255) || ((uintptr_t)cbK_packed & 15) ||
      ((uintptr_t)cbV_packed & 15))
    return LOOPVQ_ERR_INVALID_ARG;
  const WsLayout ws = decode_ws(g, layout);
  if (workspace_bytes < ws.total) return LOOPVQ_ERR_WORKSPACE_TOO_SMALL;

  const int64_t units = (int64_t)layout->batch * g.Hq;
  const DecodePlan pl = decode_plan(units, max_body_tokens(layout), device_sm_count());
  if (units > 65535LL * 65535LL || pl.max_splits > 1 << 20 || layout->batch > 65535 || g.Hq > 65535)
    return LOOPVQ_ERR_UNSUPPORTED;

  DecodeParams p;
  p.T = g.T; p.Tc = g.Tc; p.H = g.H; p.Hq = g.Hq; p.D = g.D; p.J = g.J; p.W = g.W; p.C = g.C;
  p.loop_step = loop_step;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.batch = layout->batch; p.n_sink = layout->n_sink; p.n_recent = layout->n_recent;
  p.page = layout->page; p.max_ctx = layout->max_ctx_len;
  p.ctx_len = layout->ctx_len; p.body_off = layout->body_off; p.win_off = layout->win_off;
  p.body_pool_tokens = layout->body_pool_tokens; p.win_pool_tokens = layout->win_pool_tokens;
  const size_t eb = cb_elem_bytes(g);
  const size_t slices = packed_slices_offset_bytes(g);
  const size_t step_off = slices + (size_t)loop_step * slice_elems_per_step(g) * eb;
  p.cbK_slice = (const uint8_t*)cbK_packed + step_off;
  p.cbV_slice = (const uint8_t*)cbV_packed + step_off;
  const int b_blk = loop_step / g.Tc;
  const size_t blk_bytes = (size_t)g.H * layout->body_pool_tokens * g.J;
  p.idxK = idxK_pool + b_blk * blk_bytes;
  p.idxV = idxV_pool + b_blk * blk_bytes;
  const size_t win_step = (size_t)g.H * layout->win_pool_tokens * g.D;
  p.winK = (const __nv_bfloat16*)winK + loop_step * win_step;
  p.winV = (const __nv_bfloat16*)winV + loop_step * win_step;
  p.q = q; p.q_bf16 = q_dtype == LOOPVQ_BF16;
  p.out = out; p.out_bf16 = out_dtype == LOOPVQ_BF16; p.lse = lse_out;
  p.status = (uint32_t*)workspace;
  p.tickets = (uint32_t*)((uint8_t*)workspace + ws.tickets_off);
  p.partials = (float*)((uint8_t*)workspace + ws.partials_off);
  p.split_len = pl.split_len;
  p.max_splits = pl.max_splits;

  dim3 grid(pl.max_splits, g.Hq, layout->batch);
  cudaStream_t s = (cudaStream_t)stream;
#define LOOPVQ_LAUNCH(JJ, DD, CBT)                                                                    \
  do {                                                                                               \
    auto kfn = decode_kernel<JJ, DD, CBT>;                                                           \
    if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, kDynSmem) != cudaSuccess) \
      return LOOPVQ_ERR_CUDA;                                                                        \
    kfn<<<grid, kThreads, kDynSmem, s>>>(p);                                                         \
  } while (0)
#define LOOPVQ_LAUNCH_J(DD, CBT)                      \
  do {                                                \
    if (g.J == 32) LOOPVQ_LAUNCH(32, DD, CBT);        \
    else if (g.J == 16) LOOPVQ_LAUNCH(16, DD, CBT);   \
    else LOOPVQ_LAUNCH(8, DD, CBT);                   \
  } while (0)
  if (g.D == 128) {
    if (g.cb_bf16) LOOPVQ_LAUNCH_J(128, __nv_bfloat16);
    else LOOPVQ_LAUNCH_J(128, float);
  } else {
    if (g.cb_bf16) LOOPVQ_LAUNCH_J(64, __nv_bfloat16);
    else LOOPVQ_LAUNCH_J(64, float);
  }
#undef LOOPVQ_LAUNCH_J
#undef LOOPVQ_LAUNCH
  return cudaGetLastError() == cudaSuccess ? LOOPVQ_OK : LOOPVQ_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Allocation-free variant of loopvq_decode_attn.
//
// Some callers cannot hand the library a workspace: a plugin loaded into a
// host process whose allocator owns all device memory, or a latency-critical
// path where cudaMalloc (which synchronizes the device) is not allowed.  This
// variant keeps the split partials and counters in a fixed array that lives
// in the library's own device image, so the caller supplies only inputs and
// outputs.  The array is kLoopvqStaticScratchBytes per device and stays
// resident on every GPU that loads the library until the process exits.
// ---------------------------------------------------------------------------

#include <mutex>

namespace loopvq {

constexpr size_t kLoopvqStaticScratchBytes = 8u << 20;  // 8 MiB
static __device__ __align__(256) unsigned char g_decode_scratch[kLoopvqStaticScratchBytes];

constexpr int kMaxDevices = 64;
static std::mutex g_scratch_mutex;
static void* g_scratch_addr[kMaxDevices];

// Device address of g_decode_scratch on the current device.  In host code the
// symbol is only a host-side stand-in, so the real address is looked up once
// per device (with that device current) and cached.
static loopvq_status static_scratch(void** addr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LOOPVQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return LOOPVQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return LOOPVQ_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *addr = g_scratch_addr[dev];
  return LOOPVQ_OK;
}

}  // namespace loopvq

extern "C" loopvq_status loopvq_decode_attn_noalloc(const loopvq_codebook_desc* desc, const void* cbK_packed,
                                                    const void* cbV_packed, const loopvq_cache_layout* layout,
                                                    const uint8_t* idxK_pool, const uint8_t* idxV_pool,
                                                    const void* winK, const void* winV, const void* q,
                                                    loopvq_dtype q_dtype, int32_t loop_step, float softmax_scale,
                                                    void* out, loopvq_dtype out_dtype, float* lse_out,
                                                    uint32_t* fault_bits, loopvq_stream_t stream) {
  Geo g;
  loopvq_status st = make_geo(desc, &g);
  if (st != LOOPVQ_OK) return st;
  if ((st = check_layout(layout)) != LOOPVQ_OK) return st;
  if (g.J != 8 && g.J != 16 && g.J != 32) return LOOPVQ_ERR_UNSUPPORTED;
  if (g.D != 64 && g.D != 128) return LOOPVQ_ERR_UNSUPPORTED;
  if (loop_step < 0 || loop_step >= g.T) return LOOPVQ_ERR_INVALID_ARG;
  if (q_dtype != LOOPVQ_F32 && q_dtype != LOOPVQ_BF16) return LOOPVQ_ERR_INVALID_ARG;
  if (out_dtype != LOOPVQ_F32 && out_dtype != LOOPVQ_BF16) return LOOPVQ_ERR_INVALID_ARG;
  if (!(softmax_scale == softmax_scale)) return LOOPVQ_ERR_INVALID_ARG;
  if (!cbK_packed || !cbV_packed || !idxK_pool || !idxV_pool || !winK || !winV || !q || !out)
    return LOOPVQ_ERR_INVALID_ARG;
  if (((uintptr_t)idxK_pool & 15) || ((uintptr_t)idxV_pool & 15) || ((uintptr_t)winK & 15) ||
      ((uintptr_t)winV & 15) || ((uintptr_t)cbK_packed & 15) || ((uintptr_t)cbV_packed & 15) ||
      ((uintptr_t)fault_bits & 3))
    return LOOPVQ_ERR_INVALID_ARG;
  const WsLayout ws = decode_ws(g, layout);
  if (ws.total > kLoopvqStaticScratchBytes) return LOOPVQ_ERR_WORKSPACE_TOO_SMALL;
  const int64_t units = (int64_t)layout->batch * g.Hq;
  const DecodePlan pl = decode_plan(units, max_body_tokens(layout), device_sm_count());
  if (units > 65535LL * 65535LL || pl.max_splits > 1 << 20 || layout->batch > 65535 || g.Hq > 65535)
    return LOOPVQ_ERR_UNSUPPORTED;

  void* scratch = nullptr;
  if ((st = static_scratch(&scratch)) != LOOPVQ_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  // the status word and the split counters must start at zero
  if (cudaMemsetAsync(scratch, 0, ws.partials_off, s) != cudaSuccess) return LOOPVQ_ERR_CUDA;

  DecodeParams p;
  p.T = g.T; p.Tc = g.Tc; p.H = g.H; p.Hq = g.Hq; p.D = g.D; p.J = g.J; p.W = g.W; p.C = g.C;
  p.loop_step = loop_step;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.batch = layout->batch; p.n_sink = layout->n_sink; p.n_recent = layout->n_recent;
  p.page = layout->page; p.max_ctx = layout->max_ctx_len;
  p.ctx_len = layout->ctx_len; p.body_off = layout->body_off; p.win_off = layout->win_off;
  p.body_pool_tokens = layout->body_pool_tokens; p.win_pool_tokens = layout->win_pool_tokens;
  const size_t eb = cb_elem_bytes(g);
  const size_t step_off = packed_slices_offset_bytes(g) + (size_t)loop_step * slice_elems_per_step(g) * eb;
  p.cbK_slice = (const uint8_t*)cbK_packed + step_off;
  p.cbV_slice = (const uint8_t*)cbV_packed + step_off;
  const size_t blk_bytes = (size_t)g.H * layout->body_pool_tokens * g.J;
  p.idxK = idxK_pool + (loop_step / g.Tc) * blk_bytes;
  p.idxV = idxV_pool + (loop_step / g.Tc) * blk_bytes;
  const size_t win_step = (size_t)g.H * layout->win_pool_tokens * g.D;
  p.winK = (const __nv_bfloat16*)winK + loop_step * win_step;
  p.winV = (const __nv_bfloat16*)winV + loop_step * win_step;
  p.q = q; p.q_bf16 = q_dtype == LOOPVQ_BF16;
  p.out = out; p.out_bf16 = out_dtype == LOOPVQ_BF16; p.lse = lse_out;
  p.status = fault_bits ? fault_bits : (uint32_t*)scratch;
  p.tickets = (uint32_t*)((uint8_t*)scratch + ws.tickets_off);
  p.partials = (float*)((uint8_t*)scratch + ws.partials_off);
  p.split_len = pl.split_len;
  p.max_splits = pl.max_splits;

  dim3 grid(pl.max_splits, g.Hq, layout->batch);
#define LOOPVQ_LAUNCH(JJ, DD, CBT)                                                                    \
  do {                                                                                               \
    auto kfn = decode_kernel<JJ, DD, CBT>;                                                           \
    if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, kDynSmem) != cudaSuccess) \
      return LOOPVQ_ERR_CUDA;                                                                        \
    kfn<<<grid, kThreads, kDynSmem, s>>>(p);                                                         \
  } while (0)
#define LOOPVQ_LAUNCH_J(DD, CBT)                      \
  do {                                                \
    if (g.J == 32) LOOPVQ_LAUNCH(32, DD, CBT);        \
    else if (g.J == 16) LOOPVQ_LAUNCH(16, DD, CBT);   \
    else LOOPVQ_LAUNCH(8, DD, CBT);                   \
  } while (0)
  if (g.D == 128) {
    if (g.cb_bf16) LOOPVQ_LAUNCH_J(128, __nv_bfloat16);
    else LOOPVQ_LAUNCH_J(128, float);
  } else {
    if (g.cb_bf16) LOOPVQ_LAUNCH_J(64, __nv_bfloat16);
    else LOOPVQ_LAUNCH_J(64, float);
  }
#undef LOOPVQ_LAUNCH_J
#undef LOOPVQ_LAUNCH
  return cudaGetLastError() == cudaSuccess ? LOOPVQ_OK : LOOPVQ_ERR_CUDA;
}
