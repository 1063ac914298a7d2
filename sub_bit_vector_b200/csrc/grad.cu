// Codebook gradients of the decode-attention output error (sm_100a).
//
// LoopVQ project page, "Method" -- "Component 2, Loop-aware codebook
// fine-tuning": the codebooks are tuned so that the quantized model's output
// matches the full-precision one while every loop step reads the quantized
// cache.  The stand-in objective is one attention layer: at loop step t,
//   L = weight * sum_{request, query head} || o - target ||^2
// with o the decode attention over the quantized cache (loopvq_decode_attn)
// and target the attention over the full-precision cache; the weight per step
// carries the steps' unequal sensitivity.
//
// Chain rule through softmax attention, per (request, query head), with
// g = dL/do = 2 weight (o - target) and the forward's log-sum-exp:
//   p_n   = exp(s_n - lse),       s_n  = sum_j LK[idxK[n][j]][j]
//   gv_n  = g . v_n               = sum_j LG[idxV[n][j]][j]
//   ds_n  = p_n (gv_n - g . o)    (dL/ds_n)
// where LK[c][j] = scale q_j . B^K_t[c][j] and LG[c][j] = g_j . B^V_t[c][j]
// are the per-slot tables (q_j, g_j the slot's W channels).  A body token's
// v_n and k_n channels are the codewords its codes select, so the gradients
// are per-slot histograms of the token weights times one vector each:
//   dB^V_t[c][j][w] += (sum_{n: idxV[n][j] = c} p_n)  g[jW + w]
//   dB^K_t[c][j][w] += (sum_{n: idxK[n][j] = c} ds_n) scale q[jW + w]
// Window tokens are stored in bf16 and reach no codebook entry; they enter
// only through o and lse.
//
// One CTA per (split of body tokens, query head, request): both tables and
// both histograms in shared memory ([C][J] fp32 each, code-major, so lane l
// at step s -- slot (s + l) mod J, the pool's rotated byte order -- hits bank
// (s + l) mod 32 at J = 32), lane per token over the pool's 32-token tiles,
// shared-memory float atomics for the histograms, global float atomics for
// the flush into the fp32 gradients.

#include <math.h>

#include "common.cuh"

namespace loopvq {

constexpr int kGradThreads = 256;
constexpr int kGradWarps = kGradThreads / 32;

struct GradParams {
  int T, Tc, H, Hq, D, J, W, C;
  int loop_step;
  float scale, weight;
  int batch, n_sink, n_recent, page, max_ctx;
  const int32_t* ctx_len;
  const int64_t* body_off;
  int paged;
  const int32_t* body_pages;
  int body_page_tokens, max_body_pages;
  int64_t body_pool_tokens;
  const void* cbK;   // canonical [NB][H][J][C][Tc][W]
  const void* cbV;
  int cb_bf16;
  const uint8_t* idxK;  // streams of code block t / Tc
  const uint8_t* idxV;
  const void* q;
  int q_bf16;
  const float* out;     // [batch][Hq][D] forward output
  const float* lse;     // [batch][Hq] forward log-sum-exp (natural log)
  const float* target;  // [batch][Hq][D]
  float* gradK;         // canonical, accumulated
  float* gradV;
  float* loss;          // accumulated scalar, or null
  uint32_t* faults;     // or null
  int split_len;
};

__device__ __forceinline__ float load_as_float(const void* base, int64_t e, int bf16) {
  return bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[e])
              : reinterpret_cast<const float*>(base)[e];
}

__device__ __forceinline__ void raise_fault(const GradParams& p, uint32_t bit) {
  if (p.faults) atomicOr(p.faults, bit);
}

// The J code bytes of token `lane` of a pool tile: byte s holds slot (s + lane) mod J.
template <int J>
struct TileCodes {
  uint32_t w[J / 4];
  __device__ __forceinline__ void load(const uint8_t* tile, int lane) {
    if constexpr (J == 32) {
      const uint4 a = __ldg(reinterpret_cast<const uint4*>(tile + lane * 16));
      const uint4 b = __ldg(reinterpret_cast<const uint4*>(tile + 512 + lane * 16));
      w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
      w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
    } else if constexpr (J == 16) {
      const uint4 a = __ldg(reinterpret_cast<const uint4*>(tile + lane * 16));
      w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    } else {
      const uint2 a = __ldg(reinterpret_cast<const uint2*>(tile + lane * 8));
      w[0] = a.x; w[1] = a.y;
    }
  }
  __device__ __forceinline__ int code(int s) const { return (w[s >> 2] >> ((s & 3) * 8)) & 0xff; }
};

template <int J>
__global__ void __launch_bounds__(kGradThreads) grad_kernel(const GradParams p) {
  extern __shared__ float sm[];
  float* lutK = sm;             // [256][J]
  float* lutG = lutK + 256 * J;
  float* histP = lutG + 256 * J;
  float* histS = histP + 256 * J;
  float* qs = histS + 256 * J;  // [D]
  float* gs = qs + p.D;         // [D]
  __shared__ float red[2][kGradWarps];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int split = blockIdx.x, hq = blockIdx.y, r = blockIdx.z;
  const int h = hq / (p.Hq / p.H);
  const int ctx = p.ctx_len[r];
  if (ctx < 0 || ctx > p.max_ctx) {
    if (split == 0 && tid == 0) raise_fault(p, LOOPVQ_FAULT_CTX_RANGE);
    return;
  }
  const CtxSplit cs = ctx_split(ctx, p.n_sink, p.n_recent, p.page);
  const int p0 = split * p.split_len;
  const bool has_body = p0 < cs.body;
  if (!has_body && split != 0) return;

  // q, g = 2 weight (o - target), g . o and this unit's loss
  const int64_t u = (int64_t)r * p.Hq + hq;
  float dot = 0.f, err = 0.f;
  for (int d = tid; d < p.D; d += kGradThreads) {
    const float o = p.out[u * p.D + d];
    const float diff = o - p.target[u * p.D + d];
    const float g = 2.f * p.weight * diff;
    qs[d] = load_as_float(p.q, u * p.D + d, p.q_bf16);
    gs[d] = g;
    dot = fmaf(g, o, dot);
    err = fmaf(diff, diff, err);
  }
  for (int o = 16; o; o >>= 1) {
    dot += __shfl_xor_sync(0xffffffffu, dot, o);
    err += __shfl_xor_sync(0xffffffffu, err, o);
  }
  if (lane == 0) { red[0][warp] = dot; red[1][warp] = err; }
  __syncthreads();
  float g_dot_o = 0.f, unit_err = 0.f;
  for (int w = 0; w < kGradWarps; ++w) { g_dot_o += red[0][w]; unit_err += red[1][w]; }
  if (split == 0 && tid == 0 && p.loss) atomicAdd(p.loss, p.weight * unit_err);
  if (!has_body) return;
  const int p1 = min(cs.body, p0 + p.split_len);

  // where the split's tokens sit in the pool
  int64_t first_pos = 0;
  int n_tiles;
  if (p.paged) {
    n_tiles = (p1 - p0 + 31) >> 5;
  } else {
    const int64_t off = p.body_off[r];
    if (off < 0 || off + cs.body > p.body_pool_tokens) {
      if (tid == 0) raise_fault(p, LOOPVQ_FAULT_POOL_RANGE);
      return;
    }
    first_pos = (off + p0) & ~(int64_t)31;
    n_tiles = (int)((off + p1 - first_pos + 31) >> 5);
  }

  // per-slot tables of this step's codebook slice; zeroed histograms
  const int b = p.loop_step / p.Tc, tt = p.loop_step - b * p.Tc;
  for (int e = tid; e < 256 * J; e += kGradThreads) {
    const int c = e / J, j = e - c * J;
    float k = 0.f, v = 0.f;
    if (c < p.C) {
      const int64_t base = ((((int64_t)b * p.H + h) * J + j) * p.C + c) * p.Tc * p.W + (int64_t)tt * p.W;
      for (int w = 0; w < p.W; ++w) {
        k = fmaf(qs[j * p.W + w], load_as_float(p.cbK, base + w, p.cb_bf16), k);
        v = fmaf(gs[j * p.W + w], load_as_float(p.cbV, base + w, p.cb_bf16), v);
      }
    }
    lutK[e] = p.scale * k;
    lutG[e] = v;
    histP[e] = 0.f;
    histS[e] = 0.f;
  }
  __syncthreads();

  const float lse = p.lse[u];
  const int64_t stream_base = (int64_t)h * (p.body_pool_tokens >> 5);  // idxK/idxV start at block b
  for (int i = warp; i < n_tiles; i += kGradWarps) {
    int64_t pos0;   // pool position of the tile's lane 0
    int pfirst;     // body token of lane 0
    if (p.paged) {
      pfirst = p0 + 32 * i;
      const int pg = p.body_pages[(int64_t)r * p.max_body_pages + pfirst / p.body_page_tokens];
      pos0 = (int64_t)pg * p.body_page_tokens + pfirst % p.body_page_tokens;
      if (pg < 0 || pos0 + 32 > p.body_pool_tokens) {  // whole tile lies in one page
        if (lane == 0) raise_fault(p, LOOPVQ_FAULT_POOL_RANGE);
        continue;
      }
    } else {
      pos0 = first_pos + 32 * (int64_t)i;
      pfirst = (int)(pos0 - p.body_off[r]);
    }
    const int pn = pfirst + lane;
    bool active = pn >= p0 && pn < p1;
    const int64_t tile_off = (stream_base + (pos0 >> 5)) * (32 * J);
    TileCodes<J> ck, cv;
    ck.load(p.idxK + tile_off, lane);
    cv.load(p.idxV + tile_off, lane);
    float s = 0.f, gv = 0.f;
    bool bad = false;
#pragma unroll
    for (int st = 0; st < J; ++st) {
      const int slot = (st + lane) & (J - 1);
      const int a = ck.code(st), v = cv.code(st);
      bad |= a >= p.C || v >= p.C;
      s += lutK[a * J + slot];
      gv += lutG[v * J + slot];
    }
    if (active && bad) {
      raise_fault(p, LOOPVQ_FAULT_CODE_RANGE);
      active = false;
    }
    if (!active) continue;
    const float pr = expf(s - lse);
    const float ds = pr * (gv - g_dot_o);
#pragma unroll
    for (int st = 0; st < J; ++st) {
      const int slot = (st + lane) & (J - 1);
      atomicAdd(&histP[cv.code(st) * J + slot], pr);
      atomicAdd(&histS[ck.code(st) * J + slot], ds);
    }
  }
  __syncthreads();

  // flush: histogram entry times the slot's channels of g (values) or scale q (keys)
  for (int e = tid; e < p.C * J; e += kGradThreads) {
    const float hp = histP[e], hs = histS[e];
    if (hp == 0.f && hs == 0.f) continue;
    const int c = e / J, j = e - c * J;
    const int64_t base = ((((int64_t)b * p.H + h) * J + j) * p.C + c) * p.Tc * p.W + (int64_t)tt * p.W;
    for (int w = 0; w < p.W; ++w) {
      if (hp != 0.f) atomicAdd(p.gradV + base + w, hp * gs[j * p.W + w]);
      if (hs != 0.f) atomicAdd(p.gradK + base + w, hs * p.scale * qs[j * p.W + w]);
    }
  }
}

}  // namespace loopvq

using namespace loopvq;

extern "C" loopvq_status loopvq_codebook_grad(const loopvq_codebook_desc* desc, const void* cbK, const void* cbV,
                                              const loopvq_cache_layout* layout, const uint8_t* idxK_pool,
                                              const uint8_t* idxV_pool, const void* q, loopvq_dtype q_dtype,
                                              int32_t loop_step, float softmax_scale, const float* out,
                                              const float* lse, const float* target, float weight,
                                              float* gradK, float* gradV, float* loss_out,
                                              uint32_t* fault_bits, loopvq_stream_t stream) {
  Geo g;
  loopvq_status st = make_geo(desc, &g);
  if (st != LOOPVQ_OK) return st;
  // the decode's layout validation: its workspace size is 0 for an invalid layout
  if (loopvq_decode_workspace_bytes(desc, layout) == 0) return LOOPVQ_ERR_INVALID_ARG;
  if (g.J != 8 && g.J != 16 && g.J != 32) return LOOPVQ_ERR_UNSUPPORTED;
  if (g.D != 64 && g.D != 128) return LOOPVQ_ERR_UNSUPPORTED;
  if (loop_step < 0 || loop_step >= g.T) return LOOPVQ_ERR_INVALID_ARG;
  if (q_dtype != LOOPVQ_F32 && q_dtype != LOOPVQ_BF16) return LOOPVQ_ERR_INVALID_ARG;
  if (!(softmax_scale == softmax_scale) || !(weight == weight)) return LOOPVQ_ERR_INVALID_ARG;
  if (!cbK || !cbV || !idxK_pool || !idxV_pool || !q || !out || !lse || !target || !gradK || !gradV)
    return LOOPVQ_ERR_INVALID_ARG;
  if (((uintptr_t)idxK_pool & 15) || ((uintptr_t)idxV_pool & 15)) return LOOPVQ_ERR_INVALID_ARG;
  if (layout->batch > 65535 || g.Hq > 65535) return LOOPVQ_ERR_UNSUPPORTED;

  const int64_t units = (int64_t)layout->batch * g.Hq;
  const int max_body = ctx_split(layout->max_ctx_len, layout->n_sink, layout->n_recent, layout->page).body;
  // about two CTAs per SM over all units; at least 256 tokens per split
  int64_t want = (2LL * device_sm_count() + units - 1) / units;
  const int64_t most = (max_body + 255) / 256;
  if (want > most) want = most;
  if (want < 1) want = 1;
  int split_len = (int)(((max_body + want - 1) / want + 31) & ~31LL);
  if (split_len < 32) split_len = 32;
  const int n_splits = max_body > 0 ? (max_body + split_len - 1) / split_len : 1;

  GradParams p;
  p.T = g.T; p.Tc = g.Tc; p.H = g.H; p.Hq = g.Hq; p.D = g.D; p.J = g.J; p.W = g.W; p.C = g.C;
  p.loop_step = loop_step;
  p.scale = softmax_scale;
  p.weight = weight;
  p.batch = layout->batch; p.n_sink = layout->n_sink; p.n_recent = layout->n_recent;
  p.page = layout->page; p.max_ctx = layout->max_ctx_len;
  p.ctx_len = layout->ctx_len; p.body_off = layout->body_off;
  p.paged = (layout->flags & LOOPVQ_LAYOUT_PAGED_BODY) ? 1 : 0;
  p.body_pages = layout->body_pages;
  p.body_page_tokens = p.paged ? layout->body_page_tokens : 32;
  p.max_body_pages = layout->max_body_pages;
  p.body_pool_tokens = layout->body_pool_tokens;
  p.cbK = cbK; p.cbV = cbV; p.cb_bf16 = g.cb_bf16 ? 1 : 0;
  const size_t blk_bytes = (size_t)g.H * layout->body_pool_tokens * g.J;
  p.idxK = idxK_pool + (size_t)(loop_step / g.Tc) * blk_bytes;
  p.idxV = idxV_pool + (size_t)(loop_step / g.Tc) * blk_bytes;
  p.q = q; p.q_bf16 = q_dtype == LOOPVQ_BF16;
  p.out = out; p.lse = lse; p.target = target;
  p.gradK = gradK; p.gradV = gradV; p.loss = loss_out; p.faults = fault_bits;
  p.split_len = split_len;

  const size_t smem = (size_t)4 * 256 * g.J * sizeof(float) + (size_t)2 * g.D * sizeof(float);
  dim3 grid((unsigned)n_splits, (unsigned)g.Hq, (unsigned)layout->batch);
  cudaStream_t s = (cudaStream_t)stream;
#define LOOPVQ_GRAD(JJ)                                                                                  \
  do {                                                                                                   \
    if (cudaFuncSetAttribute(grad_kernel<JJ>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != \
        cudaSuccess)                                                                                     \
      return LOOPVQ_ERR_CUDA;                                                                            \
    grad_kernel<JJ><<<grid, kGradThreads, smem, s>>>(p);                                                 \
  } while (0)
  if (g.J == 32) LOOPVQ_GRAD(32);
  else if (g.J == 16) LOOPVQ_GRAD(16);
  else LOOPVQ_GRAD(8);
#undef LOOPVQ_GRAD
  return cudaGetLastError() == cudaSuccess ? LOOPVQ_OK : LOOPVQ_ERR_CUDA;
}
