// C ABI: descriptors, status, codebook packing and index-pool conversion.
#include <math.h>

#include "common.cuh"

namespace loopvq {

loopvq_status make_geo(const loopvq_codebook_desc* d, Geo* g) {
  if (!d || !g) return LOOPVQ_ERR_INVALID_ARG;
  if (d->n_loop < 1 || d->tc < 1 || d->n_heads_kv < 1 || d->n_heads_q < 1 || d->head_dim < 1 ||
      d->group_elems < 1 || d->n_codes < 1 || d->n_codes > 256)
    return LOOPVQ_ERR_INVALID_ARG;
  if (d->cb_dtype != LOOPVQ_F32 && d->cb_dtype != LOOPVQ_BF16) return LOOPVQ_ERR_INVALID_ARG;
  if (d->n_loop % d->tc || d->group_elems % d->tc || d->n_heads_q % d->n_heads_kv) return LOOPVQ_ERR_INVALID_ARG;
  const int W = d->group_elems / d->tc;
  if (d->head_dim % W) return LOOPVQ_ERR_INVALID_ARG;
  g->T = d->n_loop;
  g->Tc = d->tc;
  g->NB = d->n_loop / d->tc;
  g->H = d->n_heads_kv;
  g->Hq = d->n_heads_q;
  g->D = d->head_dim;
  g->G = d->group_elems;
  g->W = W;
  g->J = d->head_dim / W;
  g->C = d->n_codes;
  g->cb_bf16 = d->cb_dtype == LOOPVQ_BF16;
  // pools hold 32-token tiles split into 32/J lane groups; encode keeps a
  // sub-vector in registers (G <= 64)
  if (32 % g->J || g->G > 64 || g->D > 1024) return LOOPVQ_ERR_UNSUPPORTED;
  return LOOPVQ_OK;
}

int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return 148; }
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return 148;
  }
  return n;
}

// canonical [NB][H][J][C][Tc][W] -> slices [T][H][C][J][W]
template <typename T>
__global__ void pack_slices_kernel(const T* __restrict__ can, T* __restrict__ sl, int NB, int Tc, int H, int J,
                                   int C, int W, int64_t total) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    int64_t x = e;
    const int w = (int)(x % W); x /= W;
    const int j = (int)(x % J); x /= J;
    const int c = (int)(x % C); x /= C;
    const int h = (int)(x % H); x /= H;
    const int t = (int)x;
    const int b = t / Tc, tt = t % Tc;
    sl[e] = can[((((int64_t)b * H + h) * J + j) * C + c) * Tc * W + (int64_t)tt * W + w];
  }
}

// codes [NB][H][n][J] <-> pool
__global__ void pool_pack_kernel(const uint8_t* __restrict__ codes, uint8_t* __restrict__ pool, int NB, int H, int J,
                                 int kind, int64_t n_tokens, int64_t tok_off, int64_t pool_tokens, int unpack) {
  const int64_t total = (int64_t)NB * H * n_tokens * J;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    int64_t x = e;
    const int j = (int)(x % J); x /= J;
    const int64_t n = x % n_tokens; x /= n_tokens;
    const int h = (int)(x % H);
    const int b = (int)(x / H);
    const int64_t pb = pool_byte(J, kind, pool_tokens, b, H, h, tok_off + n, j);
    if (unpack)
      const_cast<uint8_t*>(codes)[e] = pool[pb];
    else
      pool[pb] = codes[e];
  }
}

static int grid_for(int64_t total) {
  int64_t g = (total + 255) / 256;
  if (g > 148 * 32) g = 148 * 32;
  if (g < 1) g = 1;
  return (int)g;
}

}  // namespace loopvq

using namespace loopvq;

extern "C" const char* loopvq_version(void) { return "loopvq 0.1.0 sm_100a"; }

extern "C" const char* loopvq_status_string(loopvq_status s) {
  switch (s) {
    case LOOPVQ_OK: return "ok";
    case LOOPVQ_ERR_INVALID_ARG: return "invalid argument";
    case LOOPVQ_ERR_UNSUPPORTED: return "unsupported geometry";
    case LOOPVQ_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case LOOPVQ_ERR_CUDA: return "CUDA runtime error";
    case LOOPVQ_ERR_DEVICE_FAULT: return "device reported a fault";
  }
  return "unknown status";
}

extern "C" loopvq_status loopvq_validate_desc(const loopvq_codebook_desc* desc) {
  Geo g;
  loopvq_status s = make_geo(desc, &g);
  if (s != LOOPVQ_OK) return s;
  if ((g.J != 8 && g.J != 16 && g.J != 32) || g.W > 16 || (g.D != 64 && g.D != 128)) return LOOPVQ_ERR_UNSUPPORTED;
  return LOOPVQ_OK;
}

extern "C" loopvq_status loopvq_ctx_split(int32_t ctx_len, int32_t n_sink, int32_t n_recent, int32_t page,
                                         int32_t* sink, int32_t* body, int32_t* recent) {
  if (ctx_len < 0 || n_sink < 0 || n_recent < 0 || page < 1 || !sink || !body || !recent)
    return LOOPVQ_ERR_INVALID_ARG;
  const CtxSplit c = ctx_split(ctx_len, n_sink, n_recent, page);
  *sink = c.sink;
  *body = c.body;
  *recent = c.recent;
  return LOOPVQ_OK;
}

extern "C" float loopvq_bits_per_element(const loopvq_codebook_desc* desc) {
  if (!desc || desc->n_codes < 1 || desc->n_codes > 256 || desc->group_elems < 1) return -1.f;
  return log2f((float)desc->n_codes) / (float)desc->group_elems;
}

extern "C" size_t loopvq_codebook_packed_bytes(const loopvq_codebook_desc* desc) {
  Geo g;
  if (make_geo(desc, &g) != LOOPVQ_OK) return 0;
  return packed_slices_offset_bytes(g) + (size_t)g.T * slice_elems_per_step(g) * cb_elem_bytes(g);
}

extern "C" loopvq_status loopvq_codebook_pack(const loopvq_codebook_desc* desc, const void* canonical, void* packed,
                                              size_t packed_bytes, loopvq_stream_t stream) {
  Geo g;
  loopvq_status st = make_geo(desc, &g);
  if (st != LOOPVQ_OK) return st;
  if (!canonical || !packed || ((uintptr_t)packed & 15)) return LOOPVQ_ERR_INVALID_ARG;
  if (packed_bytes < loopvq_codebook_packed_bytes(desc)) return LOOPVQ_ERR_INVALID_ARG;
  const size_t eb = cb_elem_bytes(g);
  const size_t can_bytes = canonical_elems(g) * eb;
  const uint8_t* c8 = (const uint8_t*)canonical;
  uint8_t* p8 = (uint8_t*)packed;
  if (c8 < p8 + packed_bytes && p8 < c8 + can_bytes) return LOOPVQ_ERR_INVALID_ARG;  // overlap
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemcpyAsync(packed, canonical, can_bytes, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return LOOPVQ_ERR_CUDA;
  const int64_t total = (int64_t)g.T * slice_elems_per_step(g);
  void* sl = p8 + packed_slices_offset_bytes(g);
  if (g.cb_bf16)
    pack_slices_kernel<__nv_bfloat16><<<grid_for(total), 256, 0, s>>>(
        (const __nv_bfloat16*)canonical, (__nv_bfloat16*)sl, g.NB, g.Tc, g.H, g.J, g.C, g.W, total);
  else
    pack_slices_kernel<float><<<grid_for(total), 256, 0, s>>>((const float*)canonical, (float*)sl, g.NB, g.Tc, g.H,
                                                               g.J, g.C, g.W, total);
  return cudaGetLastError() == cudaSuccess ? LOOPVQ_OK : LOOPVQ_ERR_CUDA;
}

extern "C" size_t loopvq_index_pool_bytes(const loopvq_codebook_desc* desc, int64_t pool_tokens) {
  Geo g;
  if (make_geo(desc, &g) != LOOPVQ_OK || pool_tokens <= 0 || (pool_tokens & 31)) return 0;
  return (size_t)g.NB * g.H * (size_t)pool_tokens * g.J;
}

static loopvq_status pool_convert(const loopvq_codebook_desc* desc, loopvq_kind kind, const uint8_t* codes,
                                  int64_t n_tokens, const uint8_t* pool, int64_t tok_off, int64_t pool_tokens,
                                  int unpack, loopvq_stream_t stream) {
  Geo g;
  loopvq_status st = make_geo(desc, &g);
  if (st != LOOPVQ_OK) return st;
  if (kind != LOOPVQ_KEYS && kind != LOOPVQ_VALUES) return LOOPVQ_ERR_INVALID_ARG;
  if (n_tokens < 0 || tok_off < 0 || pool_tokens <= 0 || (pool_tokens & 31) || tok_off + n_tokens > pool_tokens)
    return LOOPVQ_ERR_INVALID_ARG;
  if (n_tokens == 0) return LOOPVQ_OK;
  if (!codes || !pool) return LOOPVQ_ERR_INVALID_ARG;
  const int64_t total = (int64_t)g.NB * g.H * n_tokens * g.J;
  pool_pack_kernel<<<grid_for(total), 256, 0, (cudaStream_t)stream>>>(
      codes, const_cast<uint8_t*>(pool), g.NB, g.H, g.J, (int)kind, n_tokens, tok_off, pool_tokens, unpack);
  return cudaGetLastError() == cudaSuccess ? LOOPVQ_OK : LOOPVQ_ERR_CUDA;
}

extern "C" loopvq_status loopvq_index_pool_pack(const loopvq_codebook_desc* desc, loopvq_kind kind,
                                                const uint8_t* codes, int64_t n_tokens, uint8_t* pool,
                                                int64_t tok_off, int64_t pool_tokens, loopvq_stream_t stream) {
  return pool_convert(desc, kind, codes, n_tokens, pool, tok_off, pool_tokens, 0, stream);
}

extern "C" loopvq_status loopvq_index_pool_unpack(const loopvq_codebook_desc* desc, loopvq_kind kind,
                                                  const uint8_t* pool, int64_t tok_off, int64_t pool_tokens,
                                                  int64_t n_tokens, uint8_t* codes, loopvq_stream_t stream) {
  return pool_convert(desc, kind, codes, n_tokens, pool, tok_off, pool_tokens, 1, stream);
}

extern "C" loopvq_status loopvq_read_device_status(const void* workspace, uint32_t* bits, loopvq_stream_t stream) {
  if (!workspace) return LOOPVQ_ERR_INVALID_ARG;
  uint32_t v = 0;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemcpyAsync(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess) return LOOPVQ_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return LOOPVQ_ERR_CUDA;
  if (bits) *bits = v;
  return v ? LOOPVQ_ERR_DEVICE_FAULT : LOOPVQ_OK;
}

extern "C" loopvq_status loopvq_clear_device_status(void* workspace, loopvq_stream_t stream) {
  if (!workspace) return LOOPVQ_ERR_INVALID_ARG;
  return cudaMemsetAsync(workspace, 0, sizeof(uint32_t), (cudaStream_t)stream) == cudaSuccess ? LOOPVQ_OK
                                                                                              : LOOPVQ_ERR_CUDA;
}
