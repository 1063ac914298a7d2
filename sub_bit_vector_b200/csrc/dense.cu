// Dense bf16 split-K decode attention (sm_100a): the comparator that the
// LoopVQ pages measure against (bf16 keys and values read for every token).
//
// One CTA per (split, query head, request), two CTAs per SM; each of 16
// warps streams its share of the split's tokens, 6 tokens per iteration with
// all 12 row loads in flight (about 100 KB of loads in flight per SM), and
// keeps an fp32 online softmax (log2 units); the warps merge in shared memory
// and the last split of a (request, head) merges the splits.

#include "common.cuh"

namespace loopvq {

constexpr int kDW = 16;
constexpr int kDThreads = kDW * 32;
constexpr int kDUnroll = 6;

struct DenseParams {
  int H, Hq, D, max_ctx, split_len, max_splits;
  const int32_t* ctx_len;
  const int64_t* kv_off;
  int64_t kv_pool;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const void* q;
  int q_bf16;
  float scale_log2;
  float* out;
  float* lse;
  uint32_t* status;
  uint32_t* tickets;
  float* partials;
};

template <int CPL>  // channels per lane: D / 32
__global__ void __launch_bounds__(kDThreads, 2) dense_decode_kernel(const DenseParams p) {
  __shared__ float wpart[kDW][CPL * 32 + 2];
  __shared__ float csm[2 * kMaxCombineSplits + kDThreads];
  __shared__ int flag;
  constexpr int D = CPL * 32;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, hq = blockIdx.y, r = blockIdx.z;
  const int h = hq / (p.Hq / p.H);
  const size_t unit = (size_t)r * p.Hq + hq;
  int ctx = __ldg(p.ctx_len + r);
  int64_t off = __ldg(p.kv_off + r);
  if (ctx < 0 || ctx > p.max_ctx) {
    if (tid == 0 && split == 0) set_fault(p.status, LOOPVQ_FAULT_CTX_RANGE);
    ctx = 0;
  }
  if (off < 0 || off + ctx > p.kv_pool) {
    if (tid == 0 && split == 0) set_fault(p.status, LOOPVQ_FAULT_POOL_RANGE);
    ctx = 0;
  }
  const int n_splits = (ctx + p.split_len - 1) / p.split_len;
  if (ctx == 0) {
    if (split == 0) {
      for (int d = tid; d < D; d += blockDim.x) p.out[unit * D + d] = 0.f;
      if (p.lse && tid == 0) p.lse[unit] = -INFINITY;
    }
    return;
  }
  if (split >= n_splits) return;
  const int t0 = split * p.split_len;
  const int t1 = min(ctx, t0 + p.split_len);

  float qv[CPL];
#pragma unroll
  for (int i = 0; i < CPL; ++i) {
    const size_t qi = unit * D + lane * CPL + i;
    qv[i] = (p.q_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p.q)[qi])
                      : reinterpret_cast<const float*>(p.q)[qi]) *
            p.scale_log2;
  }
  const __nv_bfloat16* kb = p.k + ((size_t)h * p.kv_pool + off) * D + lane * CPL;
  const __nv_bfloat16* vb = p.v + ((size_t)h * p.kv_pool + off) * D + lane * CPL;
  float m = -INFINITY, l = 0.f, o[CPL];
#pragma unroll
  for (int i = 0; i < CPL; ++i) o[i] = 0.f;

  for (int base = t0 + warp * kDUnroll; base < t1; base += kDW * kDUnroll) {
    float kf[kDUnroll][CPL], vf[kDUnroll][CPL];
#pragma unroll
    for (int u = 0; u < kDUnroll; ++u) {
      const int t = base + u;
      if (t < t1) {
        if constexpr (CPL == 4) {
          const uint2 a = __ldcs(reinterpret_cast<const uint2*>(kb + (size_t)t * D));
          const uint2 b = __ldcs(reinterpret_cast<const uint2*>(vb + (size_t)t * D));
          kf[u][0] = bf16_lo(a.x); kf[u][1] = bf16_hi(a.x); kf[u][2] = bf16_lo(a.y); kf[u][3] = bf16_hi(a.y);
          vf[u][0] = bf16_lo(b.x); vf[u][1] = bf16_hi(b.x); vf[u][2] = bf16_lo(b.y); vf[u][3] = bf16_hi(b.y);
        } else {
          const uint32_t a = __ldcs(reinterpret_cast<const unsigned int*>(kb + (size_t)t * D));
          const uint32_t b = __ldcs(reinterpret_cast<const unsigned int*>(vb + (size_t)t * D));
          kf[u][0] = bf16_lo(a); kf[u][1] = bf16_hi(a);
          vf[u][0] = bf16_lo(b); vf[u][1] = bf16_hi(b);
        }
      } else {
#pragma unroll
        for (int i = 0; i < CPL; ++i) kf[u][i] = vf[u][i] = 0.f;
      }
    }
    float s[kDUnroll];
#pragma unroll
    for (int u = 0; u < kDUnroll; ++u) {
      float a = 0.f;
#pragma unroll
      for (int i = 0; i < CPL; ++i) a = fmaf(qv[i], kf[u][i], a);
#pragma unroll
      for (int x = 16; x >= 1; x >>= 1) a += __shfl_xor_sync(0xffffffffu, a, x);
      s[u] = (base + u < t1) ? a : -INFINITY;
    }
    float mn = m;
#pragma unroll
    for (int u = 0; u < kDUnroll; ++u) mn = fmaxf(mn, s[u]);
    const float corr = exp2f(m - mn);
    l *= corr;
#pragma unroll
    for (int i = 0; i < CPL; ++i) o[i] *= corr;
    m = mn;
#pragma unroll
    for (int u = 0; u < kDUnroll; ++u) {
      const float pw = exp2f(s[u] - m);
      l += pw;
#pragma unroll
      for (int i = 0; i < CPL; ++i) o[i] = fmaf(pw, vf[u][i], o[i]);
    }
  }
#pragma unroll
  for (int i = 0; i < CPL; ++i) wpart[warp][lane * CPL + i] = o[i];
  if (lane == 0) { wpart[warp][D] = m; wpart[warp][D + 1] = l; }
  __syncthreads();
  float* part = p.partials + (unit * p.max_splits + split) * (size_t)(D + 4);
  float M = -INFINITY;
  for (int w = 0; w < kDW; ++w) M = fmaxf(M, wpart[w][D]);
  for (int d = tid; d < D + 2; d += blockDim.x) {
    float acc = 0.f;
    if (d != D) {
      for (int w = 0; w < kDW; ++w) {
        const float mw = wpart[w][D];
        if (mw != -INFINITY) acc += wpart[w][d] * exp2f(mw - M);
      }
    }
    part[d] = (d == D) ? M : acc;
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) flag = (atomicAdd(p.tickets + unit, 1u) == (uint32_t)(n_splits - 1)) ? 1 : 0;
  __syncthreads();
  if (flag) {
    __threadfence();
    combine_splits(p.partials + unit * p.max_splits * (size_t)(D + 4), n_splits, D, p.out + unit * D, 0,
                   p.lse ? p.lse + unit : nullptr, csm, tid, kDThreads, BlockSync{});
    if (tid == 0) atomicExch(p.tickets + unit, 0u);
  }
}

static void dense_plan(int64_t units, int max_ctx, int n_sm, int* split_len, int* max_splits) {
  int s = (int)(2 * n_sm / (units > 0 ? units : 1));  // two CTAs per SM
  const int cap = (max_ctx + 255) / 256;
  if (s > cap) s = cap;
  if (s < 1) s = 1;
  int len = (max_ctx + s - 1) / s;
  if (len < 1) len = 1;
  *split_len = len;
  *max_splits = max_ctx > 0 ? (max_ctx + len - 1) / len : 1;
}

}  // namespace loopvq

using namespace loopvq;

extern "C" size_t loopvq_dense_decode_workspace_bytes(int32_t batch, int32_t n_heads_q, int32_t head_dim,
                                                      int32_t max_ctx_len) {
  if (batch < 1 || n_heads_q < 1 || head_dim < 1 || max_ctx_len < 0) return 0;
  int len, ms;
  dense_plan((int64_t)batch * n_heads_q, max_ctx_len, 1024, &len, &ms);
  return ws_layout((int64_t)batch * n_heads_q, ms, head_dim).total;
}

extern "C" loopvq_status loopvq_dense_decode_attn(int32_t batch, int32_t n_heads_kv, int32_t n_heads_q,
                                                  int32_t head_dim, int32_t max_ctx_len, const int32_t* ctx_len,
                                                  const int64_t* kv_off, int64_t kv_pool_tokens, const void* k,
                                                  const void* v, const void* q, loopvq_dtype q_dtype,
                                                  float softmax_scale, float* out, float* lse_out, void* workspace,
                                                  size_t workspace_bytes, loopvq_stream_t stream) {
  if (batch < 1 || n_heads_kv < 1 || n_heads_q < 1 || n_heads_q % n_heads_kv || max_ctx_len < 0 ||
      kv_pool_tokens < 0)
    return LOOPVQ_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return LOOPVQ_ERR_UNSUPPORTED;
  if (q_dtype != LOOPVQ_F32 && q_dtype != LOOPVQ_BF16) return LOOPVQ_ERR_INVALID_ARG;
  if (!ctx_len || !kv_off || !k || !v || !q || !out || !workspace) return LOOPVQ_ERR_INVALID_ARG;
  if (((uintptr_t)k & 15) || ((uintptr_t)v & 15) || ((uintptr_t)workspace & 255)) return LOOPVQ_ERR_INVALID_ARG;
  const size_t need = loopvq_dense_decode_workspace_bytes(batch, n_heads_q, head_dim, max_ctx_len);
  if (workspace_bytes < need) return LOOPVQ_ERR_WORKSPACE_TOO_SMALL;
  if (batch > 65535 || n_heads_q > 65535) return LOOPVQ_ERR_UNSUPPORTED;
  const int64_t units = (int64_t)batch * n_heads_q;
  DenseParams p;
  int len, ms;
  dense_plan(units, max_ctx_len, device_sm_count(), &len, &ms);
  if (ms > kMaxCombineSplits) return LOOPVQ_ERR_UNSUPPORTED;
  const WsLayout ws = ws_layout(units, ms, head_dim);
  p.H = n_heads_kv; p.Hq = n_heads_q; p.D = head_dim; p.max_ctx = max_ctx_len;
  p.split_len = len; p.max_splits = ms;
  p.ctx_len = ctx_len; p.kv_off = kv_off; p.kv_pool = kv_pool_tokens;
  p.k = (const __nv_bfloat16*)k; p.v = (const __nv_bfloat16*)v;
  p.q = q; p.q_bf16 = q_dtype == LOOPVQ_BF16;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.out = out; p.lse = lse_out;
  p.status = (uint32_t*)workspace;
  p.tickets = (uint32_t*)((uint8_t*)workspace + ws.tickets_off);
  p.partials = (float*)((uint8_t*)workspace + ws.partials_off);
  dim3 grid(ms, n_heads_q, batch);
  if (head_dim == 128)
    dense_decode_kernel<4><<<grid, kDThreads, 0, (cudaStream_t)stream>>>(p);
  else
    dense_decode_kernel<2><<<grid, kDThreads, 0, (cudaStream_t)stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? LOOPVQ_OK : LOOPVQ_ERR_CUDA;
}
