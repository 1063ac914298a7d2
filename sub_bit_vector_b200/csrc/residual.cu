// Adjacent-loop KV-residual 4-bit quantization and decode attention (sm_100a).
//
// FlashLoop page (thelatestinai.com; "Figure 2 (c)", "Figure 3 (c-d)",
// "Table 2", "Figure 4"): the change of K/V from one loop step to the next
// gets smaller deeper in the loop, so coding each step as a residual over the
// previous step loses less than coding each step's K/V on its own; the page
// codes these residuals with 4 bits, on the axes KIVI's 4-bit quantizer uses.  Step 0 codes K_0; step t codes
// R_t = K_t - Khat_{t-1}, the residual against the previous reconstruction,
// and Khat_t = Khat_{t-1} + Q(R_t).  Q is KIVI's quantizer: 16 levels, an
// fp16 minimum and an fp16 scale per group of 32 values; keys are grouped
// per channel over 32 consecutive tokens, values per token over 32
// consecutive channels.  Every decision is taken in fp32 with separately
// rounded operations (no contraction), so the codes are reproducible bit for
// bit:  scale = (max - min) / 15, code = clamp(rint((x - min_h) / scale_h),
// 0, 15), dequant = min_h + code * scale_h.
//
// Pool layouts (pool_tokens a multiple of 32, a request's tokens start at a
// multiple of 32 so key groups are pool-aligned):
//   codes         [T][H][pool_tokens][D/2]  two codes per byte, even channel low
//   key params    [T][H][pool_tokens/32][D] half2 (min, scale)
//   value params  [T][H][pool_tokens][D/32] half2 (min, scale)
//
// Decode at loop step t streams tiles of the t+1 residual planes into shared
// memory by bulk copies (eight lanes per token, each with D/8 channels) and
// runs split-K attention with an fp32 online softmax; the last split of a
// (request, head) merges the splits.  The rebuilt key is min + code * scale
// summed over the planes, so the score q . K is
//   sum_d q_d sum_p min_p[d]  +  sum_p sum_d (q_d scale_p[d]) code_p[d]:
// from two planes on, the 8 warps sharing a key group turn q_d scale_p[d] into
// three int8 digits per channel block (under the block's own scale) once per
// tile, and each lane sums its block with dp4a over its codes expanded to
// bytes; with one plane the key row is rebuilt per element as the encoder
// did.  Values fold the same way: the weighted sum takes code * scale per
// element and the planes' minima once per token.

#include <cuda_fp16.h>
#include <math.h>

#include "common.cuh"

namespace loopvq {

constexpr int kRG = 32;  // values per quantization group

struct ResGeo {
  int T, H, Hq, D;
};

static loopvq_status res_geo(const loopvq_residual_desc* d, ResGeo* g) {
  if (!d || d->n_loop < 1 || d->n_heads_kv < 1 || d->n_heads_q < 1 || d->n_heads_q % d->n_heads_kv)
    return LOOPVQ_ERR_INVALID_ARG;
  if (d->head_dim != 64 && d->head_dim != 128) return LOOPVQ_ERR_UNSUPPORTED;
  g->T = d->n_loop;
  g->H = d->n_heads_kv;
  g->Hq = d->n_heads_q;
  g->D = d->head_dim;
  return LOOPVQ_OK;
}

// One 4-bit decision of KIVI's quantizer on x given the group's stored min
// and scale (already rounded to fp16 and back).
__device__ __forceinline__ uint32_t q4(float x, float lo, float sc) {
  if (sc == 0.f) return 0u;
  const float v = rintf(__fdiv_rn(__fsub_rn(x, lo), sc));
  return (uint32_t)fminf(fmaxf(v, 0.f), 15.f);
}
__device__ __forceinline__ float dq4(uint32_t q, float lo, float sc) { return __fadd_rn(lo, __fmul_rn((float)q, sc)); }
// Exact float of nibble i (0..7) of x, given x12 = x >> 12: nibbles 0..4 are
// read in place and 5..7 from x12 (slots 2..4).  The nibble at slot s is
// OR-ed into the mantissa of 2^(23 - 4s), whose last place at bit 4s is worth
// 1, so subtracting 2^(23 - 4s) leaves it exactly (no integer conversion).
__device__ __forceinline__ float nibf(uint32_t x, uint32_t x12, int i) {
  const int s = i <= 4 ? i : i - 3;
  const uint32_t src = i <= 4 ? x : x12;
  const uint32_t ebits = (uint32_t)(150 - 4 * s) << 23;
  return __fsub_rn(__uint_as_float((src & (0xFu << (4 * s))) | ebits), __uint_as_float(ebits));
}

struct ResEncParams {
  const void* x;
  int x_bf16;
  int64_t st, sn, sh;
  int64_t n_tokens, tok_off, pool;
  int T, H, D;
  uint8_t* codes;
  __half2* params;
};

__device__ __forceinline__ float ld_x(const ResEncParams& p, int t, int64_t n, int h, int d) {
  const int64_t e = (int64_t)t * p.st + n * p.sn + (int64_t)h * p.sh + d;
  return p.x_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p.x)[e])
                  : reinterpret_cast<const float*>(p.x)[e];
}

// Keys: one warp per (token group, head, 32-channel block); lane = channel.
// The running reconstruction of the group's 32 tokens lives in shared memory
// (lane = bank); each step reads the group twice (min/max, then codes; the
// second read hits L1).
constexpr int kREncWarps = 8;
// Each warp's passes over its 32 tokens are chains of dependent global loads:
// loops unrolled by 16 keep 16 loads in flight, and four blocks per SM bound
// the registers so that no state spills (0.66 vs 0.83 ms per 32K x 16 x 128
// x 4 tensor, the same codes and parameters).
__global__ void __launch_bounds__(kREncWarps * 32, 4) res_encode_keys(const ResEncParams p) {
  __shared__ float accs[kREncWarps][kRG][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t wid = (int64_t)blockIdx.x * kREncWarps + warp;
  const int cblocks = p.D / 32;
  const int64_t n_groups = (p.n_tokens + kRG - 1) / kRG;
  if (wid >= n_groups * p.H * cblocks) return;
  const int cb = (int)(wid % cblocks);
  const int h = (int)((wid / cblocks) % p.H);
  const int64_t g = wid / ((int64_t)cblocks * p.H);
  const int d = cb * 32 + lane;
  const int64_t n0 = g * kRG;
  const int gl = (int)min((int64_t)kRG, p.n_tokens - n0);
  float (*acc)[32] = accs[warp];
  for (int i = 0; i < kRG; ++i) acc[i][lane] = 0.f;
  const int64_t pg = (p.tok_off + n0) / kRG;  // pool group
  for (int t = 0; t < p.T; ++t) {
    float lo = INFINITY, hi = -INFINITY;
#pragma unroll 16
    for (int i = 0; i < gl; ++i) {
      const float r = __fsub_rn(ld_x(p, t, n0 + i, h, d), acc[i][lane]);
      lo = fminf(lo, r);
      hi = fmaxf(hi, r);
    }
    const __half lo_h = __float2half_rn(lo);
    const __half sc_h = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), 15.f));
    const float lo32 = __half2float(lo_h), sc32 = __half2float(sc_h);
    p.params[(((int64_t)t * p.H + h) * (p.pool / kRG) + pg) * p.D + d] = __halves2half2(lo_h, sc_h);
    uint8_t* crow = p.codes + (((int64_t)t * p.H + h) * p.pool + p.tok_off + n0) * (p.D / 2) + d / 2;
#pragma unroll 16
    for (int i = 0; i < gl; ++i) {   // gl is warp-uniform: every lane takes the shuffle
      const float r = __fsub_rn(ld_x(p, t, n0 + i, h, d), acc[i][lane]);
      const uint32_t q = q4(r, lo32, sc32);
      const uint32_t q_odd = __shfl_down_sync(0xffffffffu, q, 1);
      acc[i][lane] = __fadd_rn(acc[i][lane], dq4(q, lo32, sc32));
      if (!(lane & 1)) crow[(int64_t)i * (p.D / 2)] = (uint8_t)(q | (q_odd << 4));
    }
  }
}

// Values: one warp per (two tokens, head, 32-channel group); lane = channel,
// each group's min and max by shuffles.  The two tokens' step chains are
// independent and interleave (1.15 vs 1.30 ms per 32K x 16 x 128 x 4 tensor
// with one token per warp, the same codes and parameters; four or eight
// tokens per warp lose more to registers than they gain).
__global__ void __launch_bounds__(256) res_encode_values(const ResEncParams p) {
  const int lane = threadIdx.x & 31;
  const int64_t wid = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int cgroups = p.D / kRG;
  const int64_t n_pairs = (p.n_tokens + 1) / 2;
  if (wid >= n_pairs * p.H * cgroups) return;
  const int cg = (int)(wid % cgroups);
  const int h = (int)((wid / cgroups) % p.H);
  const int64_t n0 = 2 * (wid / ((int64_t)cgroups * p.H));
  const bool has1 = n0 + 1 < p.n_tokens;  // warp-uniform
  const int d = cg * kRG + lane;
  float acc[2] = {0.f, 0.f};
  for (int t = 0; t < p.T; ++t) {
    float r[2], lo[2], hi[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      r[u] = (u == 0 || has1) ? __fsub_rn(ld_x(p, t, n0 + u, h, d), acc[u]) : 0.f;
      lo[u] = hi[u] = r[u];
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        lo[u] = fminf(lo[u], __shfl_xor_sync(0xffffffffu, lo[u], o));
        hi[u] = fmaxf(hi[u], __shfl_xor_sync(0xffffffffu, hi[u], o));
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const __half lo_h = __float2half_rn(lo[u]);
      const __half sc_h = __float2half_rn(__fdiv_rn(__fsub_rn(hi[u], lo[u]), 15.f));
      const float lo32 = __half2float(lo_h), sc32 = __half2float(sc_h);
      const int64_t pos = p.tok_off + n0 + u;
      const uint32_t q = q4(r[u], lo32, sc32);
      const uint32_t q_odd = __shfl_down_sync(0xffffffffu, q, 1);
      acc[u] = __fadd_rn(acc[u], dq4(q, lo32, sc32));
      if (u == 0 || has1) {
        if (lane == 0) p.params[(((int64_t)t * p.H + h) * p.pool + pos) * cgroups + cg] = __halves2half2(lo_h, sc_h);
        if (!(lane & 1)) p.codes[(((int64_t)t * p.H + h) * p.pool + pos) * (p.D / 2) + d / 2] = (uint8_t)(q | (q_odd << 4));
      }
    }
  }
}

// ------------------------------------------------------------------ decode
// One CTA per (split, query head, request): a producer warp streams tiles of
// 64 tokens -- for every plane s <= t the tile's key codes, value codes, value
// parameters and key parameters -- with bulk copies (no multicast) into a
// ring of shared-memory stages; 16 consumer warps take one token per group of
// eight lanes (lane i of a group owns channels i*D/8 ..), score it from the
// staged planes (integer key digits from two planes on, the rebuilt key row
// with one plane) and keep an fp32 online softmax.
constexpr int kRW = 16;                       // consumer warps
constexpr int kRThreads = (kRW + 1) * 32;     // + the producer warp
constexpr int kRLanesPerTok = 8;
constexpr int kRTokPerWarp = 32 / kRLanesPerTok;
constexpr int kRTile = kRW * kRTokPerWarp;    // 64 tokens per stage
constexpr int kRMaxStages = 4;
constexpr int kRSmemBudget = 192 * 1024;

// bytes of one plane of one tile: key codes, value codes (64 x D/2 each),
// value parameters (64 x D/32 pairs), key parameters (2 groups x D pairs)
__host__ __device__ inline int res_plane_bytes(int D) { return 64 * D + 8 * D + 8 * D; }

struct ResDecParams {
  int T, H, Hq, D, loop_step, max_ctx, split_len, max_splits, n_stages;
  const int32_t* ctx_len;
  const int64_t* tok_off;
  int64_t pool;
  const uint8_t* ck;
  const __half2* pk;
  const uint8_t* cv;
  const __half2* pv;
  const void* q;
  int q_bf16;
  float scale_log2;
  float* out;
  float* lse;
  uint32_t* status;
  uint32_t* tickets;
  float* partials;
};

struct ResConsumerSync {
  __device__ __forceinline__ void operator()() const { asm volatile("bar.sync 1, %0;" ::"n"(kRW * 32) : "memory"); }
};

template <int CPL, bool kIntKeys>
__global__ void __launch_bounds__(kRThreads, 1) res_decode_kernel(const ResDecParams p) {
  constexpr int D = CPL * kRLanesPerTok;
  extern __shared__ __align__(128) uint8_t rsm[];
  __shared__ float wpart[kRW][D + 2];
  __shared__ float csm[2 * kMaxCombineSplits + kRW * 32];
  __shared__ __align__(8) uint64_t bars[2 * kRMaxStages];
  __shared__ int flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, hq = blockIdx.y, r = blockIdx.z;
  const int h = hq / (p.Hq / p.H);
  const size_t unit = (size_t)r * p.Hq + hq;
  int ctx = __ldg(p.ctx_len + r);
  const int64_t off = __ldg(p.tok_off + r);
  if (ctx < 0 || ctx > p.max_ctx) {
    if (tid == 0 && split == 0) set_fault(p.status, LOOPVQ_FAULT_CTX_RANGE);
    ctx = 0;
  }
  if (ctx > 0 && (off < 0 || (off % kRG) || off + ctx > p.pool)) {
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
  const int t0 = split * p.split_len;  // a multiple of 64: tiles start on key-group boundaries
  const int t1 = min(ctx, t0 + p.split_len);
  const int n_tiles = (t1 - t0 + kRTile - 1) / kRTile;
  const int planes = p.loop_step + 1;
  const int pb = res_plane_bytes(D);
  const int stage_bytes = planes * pb;
  const int NS = p.n_stages;
  uint64_t* full = bars;
  uint64_t* empty = bars + kRMaxStages;
  if (tid == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(smem_u32(full + i), 1);
      mbar_init(smem_u32(empty + i), kRW);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kRW) {  // producer
    if (lane == 0) {
      for (int i = 0; i < n_tiles; ++i) {
        const int st = i % NS;
        if (i >= NS && !mbar_wait_bounded(smem_u32(empty + st), ((i / NS) - 1) & 1)) {
          set_fault(p.status, LOOPVQ_FAULT_TIMEOUT);
          break;
        }
        const int a = t0 + i * kRTile;
        const int n = min(kRTile, t1 - a);
        const int ng = (n + kRG - 1) / kRG;        // key groups of the tile (1 or 2)
        const int nr = ng * kRG;                   // rows copied: whole groups, inside the pool
        const int64_t pos0 = off + a;
        const uint32_t bk = 32 * D, bvp = 8 * D, bkp = 8 * D;   // offsets inside a plane block
        const uint32_t bytes = (uint32_t)planes * (2u * nr * (D / 2) + nr * (D / kRG) * 4u + ng * D * 4u);
        const uint32_t fb = smem_u32(full + st);
        mbar_arrive_expect_tx(fb, bytes);
        const uint32_t sbase = smem_u32(rsm) + (uint32_t)st * stage_bytes;
        for (int s = 0; s < planes; ++s) {
          const int64_t plane = (int64_t)s * p.H + h;
          const uint32_t d0 = sbase + (uint32_t)s * pb;
          bulk_g2s(d0, p.ck + (plane * p.pool + pos0) * (D / 2), nr * (D / 2), fb);
          bulk_g2s(d0 + bk, p.cv + (plane * p.pool + pos0) * (D / 2), nr * (D / 2), fb);
          bulk_g2s(d0 + 2 * bk, p.pv + (plane * p.pool + pos0) * (D / kRG), nr * (D / kRG) * 4, fb);
          bulk_g2s(d0 + 2 * bk + bvp, p.pk + (plane * (p.pool / kRG) + pos0 / kRG) * D, ng * D * 4, fb);
          (void)bkp;
        }
      }
    }
    return;
  }

  // consumers
  const int grp = lane / kRLanesPerTok, li = lane % kRLanesPerTok;
  // The query row in log2 units, for the key-digit passes.
  float* const qs = reinterpret_cast<float*>(rsm + (size_t)NS * stage_bytes);
  int8_t* const dig = reinterpret_cast<int8_t*>(qs + D);  // [2 tile parities][2 key groups][planes][3][D]
  __shared__ float kred[2][2][8][2];                       // per parity, group, warp: max |W|, partial C
  for (int d = tid; d < D; d += kRW * 32)
    qs[d] = (p.q_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p.q)[unit * D + d])
                      : reinterpret_cast<const float*>(p.q)[unit * D + d]) *
            p.scale_log2;
  ResConsumerSync{}();
  float qv[CPL];  // the per-element key path's query channels li*CPL.. (log2 units)
#pragma unroll
  for (int c = 0; c < CPL; ++c) qv[c] = qs[li * CPL + c];
  float m = -INFINITY, l = 0.f, o[CPL];
#pragma unroll
  for (int i = 0; i < CPL; ++i) o[i] = 0.f;
  const int j = warp * kRTokPerWarp + grp;  // token of the tile
  const int gi = warp >> 3;                 // its key group within the tile (tokens 32 gi ..)
  for (int i = 0; i < n_tiles; ++i) {
    const int st = i % NS;
    if (!mbar_wait_bounded(smem_u32(full + st), (i / NS) & 1)) set_fault(p.status, LOOPVQ_FAULT_TIMEOUT);
    const int n = min(kRTile, t1 - (t0 + i * kRTile));
    const uint8_t* sb = rsm + (size_t)st * stage_bytes;
    const int par = i & 1;
    // ---- key digits of this tile's group: the score of token n is
    //   C + sum_p sum_d W_p[d] code_p[n][d],  W_p[d] = q[d] * scale_p[g][d],
    //   C = sum_d q[d] sum_p min_p[g][d].
    // Warp hw of the group's 8 writes channel block hw (the block lane hw of a
    // token scores): W over all planes as sigma (w0 + w1 / 128 + w2 / 16384)
    // with int8 digits, sigma = the block's max |W| / 127, so that the sum over
    // the block's channels runs as integer dot products.  Bytes are laid out as
    // a lane expands its codes (even nibbles, then odd ones, per 8 channels).
    if constexpr (kIntKeys) {
      const int hw = warp & 7;
      float amax = 0.f, cpart = 0.f;
      for (int e = lane; e < planes * CPL; e += 32) {
        const int s = e / CPL, d = hw * CPL + (e - s * CPL);
        const float2 kpar = __half22float2(*reinterpret_cast<const __half2*>(sb + (size_t)s * pb + 72 * D + (gi * D + d) * 4));
        amax = fmaxf(amax, fabsf(qs[d] * kpar.y));
        cpart = fmaf(qs[d], kpar.x, cpart);
      }
#pragma unroll
      for (int x = 16; x >= 1; x >>= 1) {
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, x));
        cpart += __shfl_xor_sync(0xffffffffu, cpart, x);
      }
      const float inv = amax > 0.f ? 127.f / amax : 0.f;
      for (int e = lane; e < planes * CPL; e += 32) {
        const int s = e / CPL, mm = e - s * CPL, d = hw * CPL + mm;
        const float2 kpar = __half22float2(*reinterpret_cast<const __half2*>(sb + (size_t)s * pb + 72 * D + (gi * D + d) * 4));
        const float r0 = qs[d] * kpar.y * inv;
        const float w0 = rintf(r0);
        const float r1 = (r0 - w0) * 128.f;
        const float w1 = rintf(r1);
        const float w2 = rintf((r1 - w1) * 128.f);
        const int pos = (hw * (CPL / 4) + (((mm >> 3) << 1) | (mm & 1))) * 4 + ((mm & 7) >> 1);
        int8_t* db = dig + ((size_t)((par * 2 + gi) * planes + s) * 3) * D + pos;
        db[0] = (int8_t)w0;
        db[D] = (int8_t)w1;
        db[2 * D] = (int8_t)w2;
      }
      if (lane == 0) { kred[par][gi][hw][0] = amax; kred[par][gi][hw][1] = cpart; }
      // the group's 8 warps (named barrier 2 + gi): every block's digits and
      // scale are written before any lane reads them; the tile parity keeps
      // the next tile's writes off what a slower warp may still be reading
      asm volatile("bar.sync %0, 256;" ::"r"(2 + gi) : "memory");
    }
    float v[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) v[c] = 0.f;
    int acc0 = 0, acc1 = 0, acc2 = 0;
    float k[CPL];     // the per-element key path: the token's reconstructed key channels
#pragma unroll
    for (int c = 0; c < CPL; ++c) k[c] = 0.f;
    float vlo = 0.f;  // the planes' value minima of this lane's group, added once
    for (int s = 0; s < planes; ++s) {
      const uint8_t* pl = sb + (size_t)s * pb;
      uint32_t kc[CPL / 8], vc[CPL / 8];
      if constexpr (CPL == 16) {
        const uint2 ka = *reinterpret_cast<const uint2*>(pl + j * (D / 2) + li * 8);
        const uint2 va = *reinterpret_cast<const uint2*>(pl + 32 * D + j * (D / 2) + li * 8);
        kc[0] = ka.x; kc[1] = ka.y; vc[0] = va.x; vc[1] = va.y;
      } else {
        kc[0] = *reinterpret_cast<const uint32_t*>(pl + j * (D / 2) + li * 4);
        vc[0] = *reinterpret_cast<const uint32_t*>(pl + 32 * D + j * (D / 2) + li * 4);
      }
      if constexpr (kIntKeys) {
        // codes as bytes: word 2x holds the even nibbles of code word x, 2x + 1 the odd ones
        uint32_t bw[CPL / 4];
  #pragma unroll
        for (int x = 0; x < CPL / 8; ++x) { bw[2 * x] = kc[x] & 0x0F0F0F0Fu; bw[2 * x + 1] = (kc[x] >> 4) & 0x0F0F0F0Fu; }
        const int8_t* db = dig + ((size_t)((par * 2 + gi) * planes + s) * 3) * D + li * CPL;
        uint32_t dw[3][CPL / 4];
  #pragma unroll
        for (int k = 0; k < 3; ++k) {
          if constexpr (CPL == 16) {
            const uint4 t4 = *reinterpret_cast<const uint4*>(db + k * D);
            dw[k][0] = t4.x; dw[k][1] = t4.y; dw[k][2] = t4.z; dw[k][3] = t4.w;
          } else {
            const uint2 t2 = *reinterpret_cast<const uint2*>(db + k * D);
            dw[k][0] = t2.x; dw[k][1] = t2.y;
          }
        }
  #pragma unroll
        for (int x = 0; x < CPL / 4; ++x) {
          asm("dp4a.u32.s32 %0, %1, %2, %0;" : "+r"(acc0) : "r"(bw[x]), "r"(dw[0][x]));
          asm("dp4a.u32.s32 %0, %1, %2, %0;" : "+r"(acc1) : "r"(bw[x]), "r"(dw[1][x]));
          asm("dp4a.u32.s32 %0, %1, %2, %0;" : "+r"(acc2) : "r"(bw[x]), "r"(dw[2][x]));
        }
      } else {
        // one step's residual plane: rebuild the key channels in step order
        uint32_t kc12[CPL / 8];
#pragma unroll
        for (int x = 0; x < CPL / 8; ++x) kc12[x] = kc[x] >> 12;
        const uint4* kp = reinterpret_cast<const uint4*>(pl + 72 * D + ((j / kRG) * D + li * CPL) * 4);
#pragma unroll
        for (int w = 0; w < CPL / 4; ++w) {
          const uint4 pw = kp[w];
          const uint32_t pr[4] = {pw.x, pw.y, pw.z, pw.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int c = w * 4 + u;
            const float2 kpar = __half22float2(*reinterpret_cast<const __half2*>(&pr[u]));
            k[c] = __fadd_rn(k[c], __fadd_rn(kpar.x, __fmul_rn(nibf(kc[c >> 3], kc12[c >> 3], c & 7), kpar.y)));
          }
        }
      }
      const float2 vpar =
          __half22float2(*reinterpret_cast<const __half2*>(pl + 64 * D + (j * (D / kRG) + (li * CPL) / kRG) * 4));
      vlo += vpar.x;
      uint32_t vc12[CPL / 8];
#pragma unroll
      for (int x = 0; x < CPL / 8; ++x) vc12[x] = vc[x] >> 12;
#pragma unroll
      for (int c = 0; c < CPL; ++c) v[c] = fmaf(nibf(vc[c >> 3], vc12[c >> 3], c & 7), vpar.y, v[c]);
    }
#pragma unroll
    for (int c = 0; c < CPL; ++c) v[c] += vlo;
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(empty + st));  // the warp's reads of this stage are done
    float a;
    if constexpr (kIntKeys) {
      // this lane's block: sigma_li (w0 + w1 / 128 + w2 / 16384) summed by dp4a
      a = ((float)acc0 + (float)acc1 * (1.f / 128.f) + (float)acc2 * (1.f / 16384.f)) *
          (kred[par][gi][li][0] * (1.f / 127.f));
#pragma unroll
      for (int x = kRLanesPerTok / 2; x >= 1; x >>= 1) a += __shfl_xor_sync(0xffffffffu, a, x);
      float csum = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) csum += kred[par][gi][w][1];
      a += csum;
    } else {
      a = 0.f;
#pragma unroll
      for (int c = 0; c < CPL; ++c) a = fmaf(qv[c], k[c], a);
#pragma unroll
      for (int x = kRLanesPerTok / 2; x >= 1; x >>= 1) a += __shfl_xor_sync(0xffffffffu, a, x);
    }
    const float sc = j < n ? a : -INFINITY;
    const float mn = fmaxf(m, sc);
    if (mn != -INFINITY) {
      const float corr = exp2f(m - mn);
      const float pw = exp2f(sc - mn);
      l = fmaf(l, corr, pw);
#pragma unroll
      for (int c = 0; c < CPL; ++c) o[c] = fmaf(o[c], corr, pw * v[c]);
      m = mn;
    }
  }
  // merge the warp's four token groups (lanes li, li + 8, li + 16, li + 24)
#pragma unroll
  for (int x = kRLanesPerTok; x < 32; x <<= 1) {
    const float mo = __shfl_xor_sync(0xffffffffu, m, x);
    const float lo_ = __shfl_xor_sync(0xffffffffu, l, x);
    const float mn = fmaxf(m, mo);
    const float ca = m == -INFINITY ? 0.f : exp2f(m - mn);
    const float cb = mo == -INFINITY ? 0.f : exp2f(mo - mn);
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      const float oo = __shfl_xor_sync(0xffffffffu, o[c], x);
      o[c] = o[c] * ca + oo * cb;
    }
    l = l * ca + lo_ * cb;
    m = mn;
  }
  if (grp == 0) {
#pragma unroll
    for (int c = 0; c < CPL; ++c) wpart[warp][li * CPL + c] = o[c];
    if (li == 0) { wpart[warp][D] = m; wpart[warp][D + 1] = l; }
  }
  const ResConsumerSync csync;
  csync();
  float* part = p.partials + (unit * p.max_splits + split) * (size_t)(D + 4);
  float M = -INFINITY;
  for (int w = 0; w < kRW; ++w) M = fmaxf(M, wpart[w][D]);
  for (int d = tid; d < D + 2; d += kRW * 32) {
    float acc = 0.f;
    if (d != D) {
      for (int w = 0; w < kRW; ++w) {
        const float mw = wpart[w][D];
        if (mw != -INFINITY) acc += wpart[w][d] * exp2f(mw - M);
      }
    }
    part[d] = (d == D) ? M : acc;
  }
  __threadfence();
  csync();
  if (tid == 0) flag = (atomicAdd(p.tickets + unit, 1u) == (uint32_t)(n_splits - 1)) ? 1 : 0;
  csync();
  if (flag) {
    __threadfence();
    combine_splits(p.partials + unit * p.max_splits * (size_t)(D + 4), n_splits, D, p.out + unit * D, 0,
                   p.lse ? p.lse + unit : nullptr, csm, tid, kRW * 32, csync);
    if (tid == 0) atomicExch(p.tickets + unit, 0u);
  }
}

static void res_plan(int64_t units, int max_ctx, int n_sm, int* split_len, int* max_splits) {
  int s = (int)(n_sm / (units > 0 ? units : 1));
  const int cap = (max_ctx + 255) / 256;
  if (s > cap) s = cap;
  if (s < 1) s = 1;
  int len = (max_ctx + s - 1) / s;
  len = ((len + kRTile - 1) / kRTile) * kRTile;  // tiles start on key-group boundaries
  if (len < kRTile) len = kRTile;
  *split_len = len;
  *max_splits = max_ctx > 0 ? (max_ctx + len - 1) / len : 1;
}

}  // namespace loopvq

using namespace loopvq;

extern "C" size_t loopvq_residual_codes_bytes(const loopvq_residual_desc* desc, int64_t pool_tokens) {
  ResGeo g;
  if (res_geo(desc, &g) != LOOPVQ_OK || pool_tokens <= 0 || (pool_tokens % kRG)) return 0;
  return (size_t)g.T * g.H * pool_tokens * (g.D / 2);
}

extern "C" size_t loopvq_residual_params_bytes(const loopvq_residual_desc* desc, loopvq_kind kind,
                                               int64_t pool_tokens) {
  ResGeo g;
  if (res_geo(desc, &g) != LOOPVQ_OK || pool_tokens <= 0 || (pool_tokens % kRG)) return 0;
  if (kind == LOOPVQ_KEYS) return (size_t)g.T * g.H * (pool_tokens / kRG) * g.D * sizeof(__half2);
  if (kind == LOOPVQ_VALUES) return (size_t)g.T * g.H * pool_tokens * (g.D / kRG) * sizeof(__half2);
  return 0;
}

extern "C" loopvq_status loopvq_residual_encode(const loopvq_residual_desc* desc, loopvq_kind kind, const void* x,
                                                loopvq_dtype x_dtype, int64_t n_tokens, int64_t stride_t,
                                                int64_t stride_n, int64_t stride_h, uint8_t* codes, void* params,
                                                int64_t tok_off, int64_t pool_tokens, loopvq_stream_t stream) {
  ResGeo g;
  loopvq_status st = res_geo(desc, &g);
  if (st != LOOPVQ_OK) return st;
  if (kind != LOOPVQ_KEYS && kind != LOOPVQ_VALUES) return LOOPVQ_ERR_INVALID_ARG;
  if (x_dtype != LOOPVQ_F32 && x_dtype != LOOPVQ_BF16) return LOOPVQ_ERR_INVALID_ARG;
  if (n_tokens < 0 || tok_off < 0 || (tok_off % kRG) || pool_tokens <= 0 || (pool_tokens % kRG) ||
      tok_off + n_tokens > pool_tokens)
    return LOOPVQ_ERR_INVALID_ARG;
  if (stride_t < 0 || stride_n < 0 || stride_h < 0) return LOOPVQ_ERR_INVALID_ARG;
  if (!x || !codes || !params || ((uintptr_t)params & 3)) return LOOPVQ_ERR_INVALID_ARG;
  if (n_tokens == 0) return LOOPVQ_OK;
  ResEncParams p;
  p.x = x; p.x_bf16 = x_dtype == LOOPVQ_BF16;
  p.st = stride_t; p.sn = stride_n; p.sh = stride_h;
  p.n_tokens = n_tokens; p.tok_off = tok_off; p.pool = pool_tokens;
  p.T = g.T; p.H = g.H; p.D = g.D;
  p.codes = codes; p.params = (__half2*)params;
  const int64_t warps = kind == LOOPVQ_KEYS ? ((n_tokens + kRG - 1) / kRG) * g.H * (g.D / 32)
                                            : ((n_tokens + 1) / 2) * g.H * (g.D / kRG);
  const int64_t blocks = (warps + 7) / 8;
  if (blocks > 0x7fffffffLL) return LOOPVQ_ERR_UNSUPPORTED;
  cudaStream_t s = (cudaStream_t)stream;
  if (kind == LOOPVQ_KEYS)
    res_encode_keys<<<(unsigned)blocks, kREncWarps * 32, 0, s>>>(p);
  else
    res_encode_values<<<(unsigned)blocks, 256, 0, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? LOOPVQ_OK : LOOPVQ_ERR_CUDA;
}

extern "C" size_t loopvq_residual_decode_workspace_bytes(const loopvq_residual_desc* desc, int32_t batch,
                                                         int32_t max_ctx_len) {
  ResGeo g;
  if (res_geo(desc, &g) != LOOPVQ_OK || batch < 1 || max_ctx_len < 0) return 0;
  int len, ms;
  res_plan((int64_t)batch * g.Hq, max_ctx_len, 1024, &len, &ms);
  return ws_layout((int64_t)batch * g.Hq, ms, g.D).total;
}

extern "C" loopvq_status loopvq_residual_decode_attn(const loopvq_residual_desc* desc, int32_t batch,
                                                     int32_t max_ctx_len, const int32_t* ctx_len,
                                                     const int64_t* tok_off, int64_t pool_tokens,
                                                     const uint8_t* codesK, const void* paramsK,
                                                     const uint8_t* codesV, const void* paramsV, const void* q,
                                                     loopvq_dtype q_dtype, int32_t loop_step, float softmax_scale,
                                                     float* out, float* lse_out, void* workspace,
                                                     size_t workspace_bytes, loopvq_stream_t stream) {
  ResGeo g;
  loopvq_status st = res_geo(desc, &g);
  if (st != LOOPVQ_OK) return st;
  if (batch < 1 || max_ctx_len < 0 || pool_tokens <= 0 || (pool_tokens % kRG)) return LOOPVQ_ERR_INVALID_ARG;
  if (loop_step < 0 || loop_step >= g.T) return LOOPVQ_ERR_INVALID_ARG;
  if (q_dtype != LOOPVQ_F32 && q_dtype != LOOPVQ_BF16) return LOOPVQ_ERR_INVALID_ARG;
  if (!(softmax_scale == softmax_scale)) return LOOPVQ_ERR_INVALID_ARG;
  if (!ctx_len || !tok_off || !codesK || !paramsK || !codesV || !paramsV || !q || !out || !workspace)
    return LOOPVQ_ERR_INVALID_ARG;
  if (((uintptr_t)paramsK & 15) || ((uintptr_t)paramsV & 15) || ((uintptr_t)codesK & 15) ||
      ((uintptr_t)codesV & 15) || ((uintptr_t)workspace & 255))
    return LOOPVQ_ERR_INVALID_ARG;
  if (workspace_bytes < loopvq_residual_decode_workspace_bytes(desc, batch, max_ctx_len))
    return LOOPVQ_ERR_WORKSPACE_TOO_SMALL;
  if (batch > 65535 || g.Hq > 65535) return LOOPVQ_ERR_UNSUPPORTED;
  const int64_t units = (int64_t)batch * g.Hq;
  int len, ms;
  res_plan(units, max_ctx_len, device_sm_count(), &len, &ms);
  if (ms > kMaxCombineSplits) return LOOPVQ_ERR_UNSUPPORTED;
  const WsLayout ws = ws_layout(units, ms, g.D);
  ResDecParams p;
  p.T = g.T; p.H = g.H; p.Hq = g.Hq; p.D = g.D; p.loop_step = loop_step; p.max_ctx = max_ctx_len;
  p.split_len = len; p.max_splits = ms;
  p.ctx_len = ctx_len; p.tok_off = tok_off; p.pool = pool_tokens;
  p.ck = codesK; p.pk = (const __half2*)paramsK; p.cv = codesV; p.pv = (const __half2*)paramsV;
  p.q = q; p.q_bf16 = q_dtype == LOOPVQ_BF16;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.out = out; p.lse = lse_out;
  p.status = (uint32_t*)workspace;
  p.tickets = (uint32_t*)((uint8_t*)workspace + ws.tickets_off);
  p.partials = (float*)((uint8_t*)workspace + ws.partials_off);
  const int stage_bytes = (loop_step + 1) * res_plane_bytes(g.D);
  // after the stages: the query row (D floats) and the key digits
  // (2 tile parities x 2 key groups x planes x 3 digits x D bytes)
  const int extra = g.D * 4 + 12 * (loop_step + 1) * g.D;
  int ns = (kRSmemBudget - extra) / stage_bytes;
  if (ns > kRMaxStages) ns = kRMaxStages;
  if (ns < 1) return LOOPVQ_ERR_UNSUPPORTED;   // more planes than one stage can hold
  p.n_stages = ns;
  const size_t smem = (size_t)ns * stage_bytes + extra;
  dim3 grid(ms, g.Hq, batch);
  cudaStream_t s = (cudaStream_t)stream;
  // integer key scores from two planes on; one plane keeps the per-element path
  const bool int_keys = loop_step >= 1;
  auto kfn = g.D == 128 ? (int_keys ? res_decode_kernel<16, true> : res_decode_kernel<16, false>)
                        : (int_keys ? res_decode_kernel<8, true> : res_decode_kernel<8, false>);
  if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return LOOPVQ_ERR_CUDA;
  kfn<<<grid, kRThreads, smem, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? LOOPVQ_OK : LOOPVQ_ERR_CUDA;
}
