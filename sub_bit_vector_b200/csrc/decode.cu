// Fused split-K decode attention from loop-axis VQ codes (sm_100a).
//
// LoopVQ project page, "Serving in SGLang -- Attend from indices": at loop
// step t the kernel reads keys and values from the shared index rows through
// the step's codebook slice B_t and merges them with the bf16 sink/recent
// attention.  One CTA handles one split of one (request, query head):
//
//   window split : the bf16 sink + recent tokens, online softmax in fp32.
//   body split   : up to kSplitCap tokens of codes, in two passes over a
//                  TMA-fed shared-memory ring (4 x 32 KB in flight):
//     pass K  -- score s_n = sum_j LUT[j][idxK[n][j]] with the per-step
//                lookup table LUT[j][c] = scale*log2(e) * q_j . B^K_t[c][j].
//                Lane l of a warp owns token l of a 32-token tile and walks
//                its slots in the tile's rotated order (slot (s+l) mod J at
//                step s), so every warp-wide gather hits 32 distinct banks
//                and no cross-lane reduction is needed.
//     pass V  -- with the split maximum m known, token weight
//                p_n = 2^(s_n - m) in (0, 1] becomes a u32 fixed-point
//                q_n = floor(p_n 2^S + u_n) (u_n a Weyl dither, so the
//                rounding is unbiased) and is added into a per-slot 256-bin
//                histogram hist[j][idxV[n][j]] with shared-memory integer
//                atomics (same rotation: conflict free).
//     epilogue   -- o[jW+w] = 2^-S sum_c hist[j][c] B^V_t[c][j][w].
//   Every split writes its (m, l, o); a small merge kernel, launched right
//   after as a programmatic dependent, combines them by log-sum-exp.
//
// Fixed-point bound: a split holds n <= 8192 = 2^13 tokens and S = clz(n),
// so n * (2^S + 1) < 2^32: no bin or sum can overflow.

#include <math.h>
#include <stdio.h>

#include <utility>

#include "common.cuh"

namespace loopvq {

constexpr int kNW = 16;                      // consumer warps
constexpr int kThreads = (kNW + 1) * 32;     // + one producer warp
constexpr int kStageBytes = 32768;
// Ring depth and split cap.  When the value slice fits two stages (bf16 at
// D = 128, either type at D = 64) the ring has three stages and splits of up
// to 8192 tokens (a 32 KB score buffer): a 64K context needs 8 splits per
// head instead of 17 and fits one wave on 148 SMs, and long batched contexts
// pay the per-split start-up and epilogue half as often.  An fp32 slice at
// D = 128 takes four stages, which leaves 16 KB of scores: 4064 tokens.
// With static inputs a CTA streams its first ring-full of chunks before the
// previous kernel has finished; the producer waits for that kernel before it
// waits for a stage to drain (the consumers only start after it).
constexpr int kSplitCap = 4064;              // default max body tokens per split, multiple of 32
constexpr int kSplitCapLong = 8192;
constexpr bool long_splits(int D, int cb_bytes) { return 256 * D * cb_bytes <= 2 * kStageBytes; }
template <int J, int D, typename CBT>
struct Ring {
  static constexpr bool kLong = long_splits(D, (int)sizeof(CBT));
  static constexpr int kStages = kLong ? 3 : 4;
  static constexpr int kCap = kLong ? kSplitCapLong : kSplitCap;
};
// One 64 KB region of 256 rows (one per code) of 64 four-byte columns holds
// the lookup table during pass K and the histogram during pass V.  Column x
// stands for slot x mod J (the table is replicated 64/J times), so lane l at
// step s uses column l + s: 32 distinct banks, no wrap-around.  The region is
// 64 KB aligned in the shared window, so the address of (code, column l) is a
// single byte permute (code in byte 1, l*4 in byte 0, the region base in
// bytes 2-3) and the step's 4*s is the load's immediate offset.
constexpr int kRegionBytes = 65536;
constexpr int kCols = 64;
constexpr int kMiscBytes = 4096;
// allocation: the region, the ring, scores and misc, plus room to align the
// region to 64 KB (the part below the region holds misc, scores and ring
// stages that fit there)
constexpr int kDynSmem = 228352;

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
  float* partials;
  // Several loop steps in one launch: step loop_step + i for i < n_steps;
  // queries, outputs, lse and partials are [n_steps][batch][Hq]..., the
  // codebook slices and window pools advance by a step's size, the index
  // pools by a code block's.
  int n_steps;
  int64_t slice_step_elems, win_step_elems, idx_blk_bytes;
  int split_len;   // body tokens per split (multiple of 32, <= the kernel's cap)
  int max_splits;  // grid.x
  int static_inputs;  // layout arrays, index pools and codebooks are not being written by earlier kernels
  // paged body: body token p at pool position body_pages[r][p / bpt] * bpt + p % bpt
  int paged;
  const int32_t* body_pages;
  int body_page_tokens, max_body_pages;
  // ring window: recent token k at win_off + n_sink + (win_head + k) % win_ring
  int ring;
  const int32_t* win_head;
  int win_ring;
  // the current token's K and V of this step ([batch][H][D] bf16), or null
  const __nv_bfloat16* new_k;
  const __nv_bfloat16* new_v;
};

// Window-pool row of window token i (sink tokens first, then the recent ones
// oldest first).
__device__ __forceinline__ int64_t win_row(const DecodeParams& p, int64_t win_off, int sink, int whead, int i) {
  if (!p.ring || i < sink) return win_off + i;
  return win_off + p.n_sink + (whead + (i - sink)) % p.win_ring;
}
// Rows i .. i+len-1 that are contiguous in the pool, starting at window token i.
__device__ __forceinline__ int win_run(const DecodeParams& p, int sink, int whead, int i, int end) {
  if (!p.ring) return end - i;
  if (i < sink) return min(end, sink) - i;
  const int slot = (whead + (i - sink)) % p.win_ring;
  return min(end - i, p.win_ring - slot);
}

// Programmatic dependent launch: the kernel is launched so that it may start
// while the previous kernel in the stream finishes.  Everything that kernel
// may write (queries, windows, outputs, workspace, and -- unless the caller
// vouches for them -- layout arrays and index pools) is touched only after
// griddep_wait().  Codebooks are always treated as constant.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kNW * 32) : "memory");
}

__device__ __forceinline__ float lds_f32(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
  return v;
}
template <int OFF>
__device__ __forceinline__ float lds_f32_off(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1+%2];" : "=f"(v) : "r"(a), "n"(OFF));
  return v;
}
template <int OFF>
__device__ __forceinline__ void red_u32_off(uint32_t a, uint32_t v) {
  asm volatile("red.shared.add.u32 [%0+%1], %2;" ::"r"(a), "n"(OFF), "r"(v) : "memory");
}
// acc (two packed fp32) += (x, y)
__device__ __forceinline__ uint64_t add_f32x2(uint64_t acc, float x, float y) {
  uint64_t r;
  asm("{\n .reg .b64 t;\n mov.b64 t, {%2, %3};\n add.rn.f32x2 %0, %1, t;\n}" : "=l"(r) : "l"(acc), "f"(x), "f"(y));
  return r;
}
__device__ __forceinline__ float sum_f32x2(uint64_t a) {
  return __uint_as_float((uint32_t)a) + __uint_as_float((uint32_t)(a >> 32));
}
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// This lane's J code bytes of a tile (see the tile layout in common.cuh).
template <int J>
__device__ __forceinline__ void load_tile_words(const uint8_t* tile, int lane, uint32_t (&w)[J / 4]) {
  if constexpr (J == 32) {
    const uint4 a = *reinterpret_cast<const uint4*>(tile + lane * 16);
    const uint4 b = *reinterpret_cast<const uint4*>(tile + 512 + lane * 16);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
  } else if constexpr (J == 16) {
    const uint4 a = *reinterpret_cast<const uint4*>(tile + lane * 16);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
  } else {
    const uint2 a = *reinterpret_cast<const uint2*>(tile + lane * 8);
    w[0] = a.x; w[1] = a.y;
  }
}

// Shared address of (code = byte K of w, column lane): lb holds the region
// base (bytes 2-3) and lane*4 (byte 0); the code becomes byte 1.
template <int K>
__device__ __forceinline__ uint32_t code_addr(uint32_t w, uint32_t lb) {
  return __byte_perm(w, lb, 0x7604u | (K << 4));
}

// Word I of a lane's codes (steps 4I .. 4I+3) for two tiles: gathers of
// table columns lane + s (immediate offset 4s) into packed fp32 pair sums.
template <int I>
__device__ __forceinline__ void score_word(uint32_t w0, uint32_t w1, uint32_t lb, uint64_t& a01, uint64_t& a23,
                                           uint64_t& b01, uint64_t& b23) {
  const float x0 = lds_f32_off<16 * I + 0>(code_addr<0>(w0, lb));
  const float y0 = lds_f32_off<16 * I + 0>(code_addr<0>(w1, lb));
  const float x1 = lds_f32_off<16 * I + 4>(code_addr<1>(w0, lb));
  const float y1 = lds_f32_off<16 * I + 4>(code_addr<1>(w1, lb));
  const float x2 = lds_f32_off<16 * I + 8>(code_addr<2>(w0, lb));
  const float y2 = lds_f32_off<16 * I + 8>(code_addr<2>(w1, lb));
  const float x3 = lds_f32_off<16 * I + 12>(code_addr<3>(w0, lb));
  const float y3 = lds_f32_off<16 * I + 12>(code_addr<3>(w1, lb));
  a01 = add_f32x2(a01, x0, x1);
  b01 = add_f32x2(b01, y0, y1);
  a23 = add_f32x2(a23, x2, x3);
  b23 = add_f32x2(b23, y2, y3);
}
template <int N, int... Is>
__device__ __forceinline__ void score_words(const uint32_t (&w0)[N], const uint32_t (&w1)[N], uint32_t lb,
                                            uint64_t& a01, uint64_t& a23, uint64_t& b01, uint64_t& b23,
                                            std::integer_sequence<int, Is...>) {
  (score_word<Is>(w0[Is], w1[Is], lb, a01, a23, b01, b23), ...);
}

// Scores of this lane's token in two tiles at once (two independent chains
// for latency hiding): the sum over its J codes of table column lane + s at
// step s, i.e. slot (s + lane) mod J, which is the tile's byte order.
template <int J>
__device__ __forceinline__ void score_pair(const uint32_t (&w0)[J / 4], const uint32_t (&w1)[J / 4], uint32_t lb,
                                           float& s0, float& s1) {
  uint64_t a01 = 0, a23 = 0, b01 = 0, b23 = 0;   // packed fp32 pairs, 0 bits = (0, 0)
  score_words(w0, w1, lb, a01, a23, b01, b23, std::make_integer_sequence<int, J / 4>{});
  s0 = sum_f32x2(a01) + sum_f32x2(a23);
  s1 = sum_f32x2(b01) + sum_f32x2(b23);
}

template <int I>
__device__ __forceinline__ void hist_word(uint32_t w0, uint32_t w1, uint32_t lb, uint32_t q0, uint32_t q1) {
  red_u32_off<16 * I + 0>(code_addr<0>(w0, lb), q0);
  red_u32_off<16 * I + 0>(code_addr<0>(w1, lb), q1);
  red_u32_off<16 * I + 4>(code_addr<1>(w0, lb), q0);
  red_u32_off<16 * I + 4>(code_addr<1>(w1, lb), q1);
  red_u32_off<16 * I + 8>(code_addr<2>(w0, lb), q0);
  red_u32_off<16 * I + 8>(code_addr<2>(w1, lb), q1);
  red_u32_off<16 * I + 12>(code_addr<3>(w0, lb), q0);
  red_u32_off<16 * I + 12>(code_addr<3>(w1, lb), q1);
}
template <int N, int... Is>
__device__ __forceinline__ void hist_words(const uint32_t (&w0)[N], const uint32_t (&w1)[N], uint32_t lb, uint32_t q0,
                                           uint32_t q1, std::integer_sequence<int, Is...>) {
  (hist_word<Is>(w0[Is], w1[Is], lb, q0, q1), ...);
}

// Adds this lane's token weights of two tiles into the histogram bins of
// their codes (same columns as the scores).
template <int J>
__device__ __forceinline__ void hist_pair(const uint32_t (&w0)[J / 4], const uint32_t (&w1)[J / 4], uint32_t lb,
                                          uint32_t q0, uint32_t q1) {
  hist_words(w0, w1, lb, q0, q1, std::make_integer_sequence<int, J / 4>{});
}

// Loads W consecutive codebook elements (bf16 or fp32) as fp32; zero if !ok.
template <int W, typename CBT>
__device__ __forceinline__ void load_vec(const CBT* p, bool ok, float (&v)[W]) {
  if constexpr (sizeof(CBT) == 2) {
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

// kSteps: a launch of several loop steps (the single-step instance keeps the
// step index a compile-time zero and its registers to itself).
template <int J, int D, typename CBT, bool kSteps>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const DecodeParams p) {
  extern __shared__ __align__(1024) uint8_t dyn[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // Query head fastest, the window split last: CTAs are dispatched in this
  // order, so the light window splits take the SMs that the previous launch
  // frees last and every body split starts (and prefetches) as early as it can.
  // The steps of one (query head, split) are adjacent in x, so they run side
  // by side and share each index row through L2.
  const int hq = kSteps ? (int)(blockIdx.x / p.n_steps) : (int)blockIdx.x;
  const int split = blockIdx.y, r = blockIdx.z;
  auto step_index = [&]() -> int { return kSteps ? (int)(blockIdx.x - (blockIdx.x / p.n_steps) * p.n_steps) : 0; };
  const int group = p.Hq / p.H;
  const int h = hq / group;
  constexpr int W = D / J;
  constexpr int kPer = 256 * J / (kNW * 32);   // lookup-table entries per consumer thread
  constexpr int kStages = Ring<J, D, CBT>::kStages;
  constexpr int kScoresBytes = Ring<J, D, CBT>::kCap * 4;

  griddep_launch_dependents();
  if (!p.static_inputs) griddep_wait();

  // ---- loads that depend only on the block index, all issued up front ----
  int ctx = __ldg(p.ctx_len + r);
  const int64_t body_off = __ldg(p.body_off + r);
  const int64_t win_off = __ldg(p.win_off + r);
  const size_t unit = ((size_t)step_index() * p.batch + r) * p.Hq + hq;
  // The query row is read right after the dependency resolves; pulling its
  // lines into L2 now (a hint: L2 stays coherent with the previous kernel's
  // writes) takes the DRAM latency off that critical step.
  if (p.static_inputs && tid < (D * (p.q_bf16 ? 2 : 4)) / 128) {
    const char* qrow = reinterpret_cast<const char*>(p.q) + unit * D * (p.q_bf16 ? 2 : 4);
    asm volatile("prefetch.global.L2 [%0];" ::"l"(qrow + tid * 128));
  }
  float wk[kPer][W];               // B^K_t entries (c, j) = tid + 512k, code-major slice
  const CBT* bk = reinterpret_cast<const CBT*>(p.cbK_slice) + step_index() * p.slice_step_elems + (size_t)h * p.C * J * W;
  if (tid < kNW * 32) {
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const int e = tid + k * kNW * 32;
      load_vec<W>(bk + (size_t)e * W, e / J < p.C, wk[k]);
    }
  }

  // ---- work of this CTA -------------------------------------------------
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
  if (ctx == 0) return;  // empty context: the merge kernel writes a zero output
  if (split >= n_splits) return;
  const bool is_window = has_win && split == n_body_splits;  // partial row n_body_splits
  const int bsplit = split;
  const int whead = (is_window && p.ring) ? __ldg(p.win_head + r) : 0;
  if (is_window) {
    if (p.ring) {
      if (win_off < 0 || win_off + p.n_sink + p.win_ring > p.win_pool_tokens || whead < 0 || whead >= p.win_ring)
        bad = true;
    } else if (win_off < 0 || win_off + n_win > p.win_pool_tokens) {
      bad = true;
    }
  } else if (!p.paged) {
    if (body_off < 0 || (body_off & 31) || body_off + cs.body > p.body_pool_tokens) bad = true;
  }
  if (bad && tid == 0) set_fault(p.status, LOOPVQ_FAULT_POOL_RANGE);
  const int tok0 = is_window ? 0 : bsplit * p.split_len;
  const int n_tok = bad ? 0 : (is_window ? n_win : min(p.split_len, cs.body - tok0));
  const int n_tiles = (n_tok + 31) >> 5;

  // ---- shared memory ------------------------------------------------------
  // 64 KB-aligned [code][table | histogram] region; misc, scores and ring
  // stages go below it while they fit, the rest above it.
  const uint32_t sbase = smem_u32(dyn);
  const uint32_t region = (sbase + (kRegionBytes - 1)) & ~(uint32_t)(kRegionBytes - 1);
  uint32_t lo = sbase, hi = region + kRegionBytes;
  auto place = [&](uint32_t bytes) -> uint32_t {
    if (lo + bytes <= region) { const uint32_t a = lo; lo += bytes; return a; }
    const uint32_t a = hi; hi += bytes; return a;
  };
  const uint32_t misc_a = place(kMiscBytes);
  const uint32_t sc_a = place(kScoresBytes);
  // The three-stage ring is one block (stage i at ring_a + i * kStageBytes);
  // the four-stage ring puts one stage below the region.
  uint32_t stage_a[kStages];
  if constexpr (Ring<J, D, CBT>::kLong) {
    const uint32_t ring_a = place(kStages * kStageBytes);
#pragma unroll
    for (int i = 0; i < kStages; ++i) stage_a[i] = ring_a + i * kStageBytes;
  } else {
#pragma unroll
    for (int i = 0; i < kStages; ++i) stage_a[i] = place(kStageBytes);
  }
  if (hi > sbase + kDynSmem) {  // cannot happen with the 1 KB reserved window start
    if (tid == 0) set_fault(p.status, LOOPVQ_FAULT_TIMEOUT);
    return;
  }
  uint8_t* const region_p = dyn + (region - sbase);
  float* const lut = reinterpret_cast<float*>(region_p);         // pass K: lut[c*64 + col]
  uint32_t* const hist = reinterpret_cast<uint32_t*>(region_p);  // pass V: hist[c*64 + col]
  auto stage_ptr = [&](int i) -> uint8_t* {
    if constexpr (Ring<J, D, CBT>::kLong) return dyn + (stage_a[0] - sbase) + i * kStageBytes;
    else return dyn + (stage_a[i] - sbase);
  };
  float* const sc = reinterpret_cast<float*>(dyn + (sc_a - sbase));
  uint8_t* const misc = dyn + (misc_a - sbase);
  uint64_t* const full_bar = reinterpret_cast<uint64_t*>(misc);
  uint64_t* const empty_bar = full_bar + kStages;
  float* const red = reinterpret_cast<float*>(misc + 256);          // [kNW * 2]

  // chunks: window -> K rows then V rows, kRowsPerChunk tokens each;
  //         body   -> K tiles then V tiles, kTilesPerChunk each.
  constexpr int kTilesPerChunk = kStageBytes / (32 * J);
  constexpr int kRowsPerChunk = kStageBytes / (D * 2);
  const int n_chunks_half = is_window ? (n_tok + kRowsPerChunk - 1) / kRowsPerChunk
                                      : (n_tiles + kTilesPerChunk - 1) / kTilesPerChunk;
  const int n_chunks = 2 * n_chunks_half;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(full_bar + s), 1);
      mbar_init(smem_u32(empty_bar + s), kNW);
    }
    fence_mbar_init();
  }
  __syncthreads();

  // ======================= producer warp ===================================
  // All 32 lanes walk the chunks (they hold a window of the page table for
  // the paged body); lane 0 issues the barrier operations and the copies.
  if (warp == kNW) {
    const bool leader = lane == 0;
    const int sidx = step_index();
    const uint8_t* vslice = reinterpret_cast<const uint8_t*>(p.cbV_slice) +
                            (sidx * p.slice_step_elems + (size_t)h * p.C * D) * sizeof(CBT);
    const int64_t idx_blk = (int64_t)((p.loop_step + sidx) / p.Tc - p.loop_step / p.Tc) * p.idx_blk_bytes;
    const uint32_t vslice_bytes = (uint32_t)(p.C * D * sizeof(CBT));
    if (leader && !is_window && n_tok > 0) prefetch_l2(vslice, vslice_bytes);  // the epilogue's codebook slice
    // window rows may be written by the kernels before this one (an earlier
    // decode call of the same cache stores its new token there)
    if (is_window && p.static_inputs) griddep_wait();
    const int n_slice = (is_window || n_tok == 0) ? 0 : (int)((vslice_bytes + kStageBytes - 1) / kStageBytes);
    const int32_t* pages = p.paged ? p.body_pages + (size_t)r * p.max_body_pages : nullptr;
    const int64_t n_phys = p.paged ? p.body_pool_tokens / p.body_page_tokens : 0;
    int pbase = -1 << 30, pcache = -1;  // page ids pbase + lane
    for (int k = 0; k < n_chunks + n_slice; ++k) {
      const int s = k % kStages;
      if (k == kStages && p.static_inputs) griddep_wait();
      if (k >= kStages) {
        int ok = 1;
        if (leader) ok = mbar_wait_bounded(smem_u32(empty_bar + s), ((k / kStages) - 1) & 1) ? 1 : 0;
        if (!__shfl_sync(0xffffffffu, ok, 0)) {
          if (leader) set_fault(p.status, LOOPVQ_FAULT_TIMEOUT);
          break;
        }
      }
      const uint32_t dst = Ring<J, D, CBT>::kLong ? stage_a[0] + (uint32_t)s * kStageBytes : stage_a[s];
      const uint32_t fb = smem_u32(full_bar + s);
      if (k >= n_chunks) {  // a piece of the value codebook slice, for the epilogue
        const uint32_t off = (uint32_t)(k - n_chunks) * kStageBytes;
        const uint32_t bytes = min((uint32_t)kStageBytes, vslice_bytes - off);
        if (leader) {
          mbar_arrive_expect_tx(fb, bytes);
          bulk_g2s(dst, vslice + off, bytes, fb);
        }
      } else if (is_window) {
        const bool vpass = k >= n_chunks_half;
        const int t0 = (vpass ? k - n_chunks_half : k) * kRowsPerChunk;
        const int t1 = min(n_tok, t0 + kRowsPerChunk);
        const __nv_bfloat16* base = (vpass ? p.winV : p.winK) + sidx * p.win_step_elems + (size_t)h * p.win_pool_tokens * D;
        if (leader) {
          mbar_arrive_expect_tx(fb, (uint32_t)(t1 - t0) * D * 2);
          for (int i = t0; i < t1;) {  // contiguous runs of rows (a ring wraps once at most)
            const int len = win_run(p, cs.sink, whead, i, t1);
            bulk_g2s(dst + (uint32_t)(i - t0) * D * 2, base + win_row(p, win_off, cs.sink, whead, i) * D,
                     (uint32_t)len * D * 2, fb);
            i += len;
          }
        }
      } else {
        const bool vpass = k >= n_chunks_half;
        const int c = vpass ? k - n_chunks_half : k;
        const int tl0 = c * kTilesPerChunk;
        const int nt = min(kTilesPerChunk, n_tiles - tl0);
        const uint8_t* stream = (vpass ? p.idxV : p.idxK) + idx_blk + (int64_t)h * (p.body_pool_tokens >> 5) * (32 * J);
        if (!p.paged) {
          if (leader) {
            const int64_t tile = ((body_off + tok0) >> 5) + tl0;
            mbar_arrive_expect_tx(fb, (uint32_t)nt * 32 * J);
            bulk_g2s(dst, stream + tile * (32 * J), (uint32_t)nt * 32 * J, fb);
          }
        } else {
          // logical body tokens [a, e) split at page boundaries; invalid pages
          // are reported and skipped (their bytes are not expected)
          const int a = tok0 + tl0 * 32, e = a + nt * 32;
          const int bpt = p.body_page_tokens;
          uint32_t valid = 0;
          for (int pass = 0; pass < 2; ++pass) {
            if (pass == 1 && leader) mbar_arrive_expect_tx(fb, valid);
            for (int t = a; t < e;) {
              const int pi = t / bpt;
              const int len = min(e - t, bpt - t % bpt);
              if (pi < pbase || pi >= pbase + 32) {  // warp-uniform
                pbase = pi;
                pcache = pbase + lane < p.max_body_pages ? __ldg(pages + pbase + lane) : -1;
              }
              const int phys = __shfl_sync(0xffffffffu, pcache, pi - pbase);
              const bool ok = pi < p.max_body_pages && phys >= 0 && phys < n_phys;
              if (pass == 0) {
                if (ok) valid += (uint32_t)len * J;
                else if (leader) set_fault(p.status, LOOPVQ_FAULT_POOL_RANGE);
              } else if (ok && leader) {
                const int64_t pos = (int64_t)phys * bpt + t % bpt;  // a multiple of 32
                bulk_g2s(dst + (uint32_t)(t - a) * J, stream + (pos >> 5) * (32 * J), (uint32_t)len * J, fb);
              }
              t += len;
            }
          }
        }
      }
    }
    return;
  }

  // ======================= consumer warps ==================================
  if (p.static_inputs) griddep_wait();  // queries, windows, workspace and outputs from here on
  float* const part = p.partials + (unit * p.max_splits + split) * (size_t)(D + 4);
  const int ctid = tid;  // 0 .. kNW*32-1

  if (is_window) {
    // Two passes over the bf16 rows: scores of every window token (lanes own
    // channels lane*CPL.., four tokens per warp in flight), the window max,
    // then the weighted sum of the value rows.
    constexpr int CPL = D >> 5;
    float qv[CPL], ov[CPL];
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
      qv[i] = load_q(p.q, p.q_bf16, unit * D + lane * CPL + i) * p.scale_log2;
      ov[i] = 0.f;
    }
    // The current token is the last window token.  With new_k/new_v given,
    // its row in the stage is replaced by them (the pool row may not hold it
    // yet), and one CTA per KV head also stores them into the window pool.
    const int i_cur = n_tok - 1;
    const bool has_new = p.new_k != nullptr && n_tok > 0;
    if (has_new && hq % group == 0 && warp == 0) {
      const int64_t row = win_row(p, win_off, cs.sink, whead, i_cur);
      const int sidx = step_index();
      const size_t src = (((size_t)sidx * p.batch + r) * p.H + h) * D + lane * CPL;
      const size_t dstp = ((size_t)h * p.win_pool_tokens + row) * D + lane * CPL;
      __nv_bfloat16* wk = const_cast<__nv_bfloat16*>(p.winK) + sidx * p.win_step_elems;
      __nv_bfloat16* wv = const_cast<__nv_bfloat16*>(p.winV) + sidx * p.win_step_elems;
#pragma unroll
      for (int i = 0; i < CPL; ++i) {
        wk[dstp + i] = p.new_k[src + i];
        wv[dstp + i] = p.new_v[src + i];
      }
    }
    // overwrite row i_cur - t0 of a stage that holds window tokens from t0
    auto patch_row = [&](uint8_t* st, int t0, const __nv_bfloat16* nv) {
      if (warp == 0) {
        const __nv_bfloat16* src = nv + (((size_t)step_index() * p.batch + r) * p.H + h) * D + lane * CPL;
        __nv_bfloat16* d = reinterpret_cast<__nv_bfloat16*>(st + (size_t)(i_cur - t0) * D * 2) + lane * CPL;
#pragma unroll
        for (int i = 0; i < CPL; ++i) d[i] = src[i];
        fence_proxy_async();  // the stage is refilled by TMA later
      }
      consumer_sync();
    };
    float mx = -INFINITY;
    for (int k = 0; k < n_chunks_half; ++k) {
      const int s = k % kStages;
      if (!mbar_wait_bounded(smem_u32(full_bar + s), (k / kStages) & 1)) set_fault(p.status, LOOPVQ_FAULT_TIMEOUT);
      const uint8_t* st = stage_ptr(s);
      const int nt = min(kRowsPerChunk, n_tok - k * kRowsPerChunk);
      if (has_new && i_cur / kRowsPerChunk == k) patch_row(stage_ptr(s), k * kRowsPerChunk, p.new_k);
      for (int b0 = warp; b0 < nt; b0 += 4 * kNW) {
        float dot[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int tkn = b0 + u * kNW < nt ? b0 + u * kNW : b0;
          const uint8_t* kr = st + (size_t)tkn * D * 2 + lane * CPL * 2;
          float kf[CPL];
          if constexpr (CPL == 4) {
            const uint2 a = *reinterpret_cast<const uint2*>(kr);
            kf[0] = bf16_lo(a.x); kf[1] = bf16_hi(a.x); kf[2] = bf16_lo(a.y); kf[3] = bf16_hi(a.y);
          } else {
            const uint32_t a = *reinterpret_cast<const uint32_t*>(kr);
            kf[0] = bf16_lo(a); kf[1] = bf16_hi(a);
          }
          dot[u] = 0.f;
#pragma unroll
          for (int i = 0; i < CPL; ++i) dot[u] = fmaf(qv[i], kf[i], dot[u]);
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
#pragma unroll
          for (int u = 0; u < 4; ++u) dot[u] += __shfl_xor_sync(0xffffffffu, dot[u], o);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int tkn = b0 + u * kNW;
          if (tkn < nt) {
            if (lane == u) sc[k * kRowsPerChunk + tkn] = dot[u];
            mx = fmaxf(mx, dot[u]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(empty_bar + s));
    }
    if (lane == 0) red[warp] = mx;
    consumer_sync();
    float m = -INFINITY;
    for (int w = 0; w < kNW; ++w) m = fmaxf(m, red[w]);
    float l = 0.f;
    for (int k = n_chunks_half; k < n_chunks; ++k) {
      const int s = k % kStages;
      if (!mbar_wait_bounded(smem_u32(full_bar + s), (k / kStages) & 1)) set_fault(p.status, LOOPVQ_FAULT_TIMEOUT);
      const uint8_t* st = stage_ptr(s);
      const int kv = k - n_chunks_half;
      const int nt = min(kRowsPerChunk, n_tok - kv * kRowsPerChunk);
      if (has_new && i_cur / kRowsPerChunk == kv) patch_row(stage_ptr(s), kv * kRowsPerChunk, p.new_v);
      for (int tkn = warp; tkn < nt; tkn += kNW) {
        const float pw = exp2f(sc[kv * kRowsPerChunk + tkn] - m);
        const uint8_t* vr = st + (size_t)tkn * D * 2 + lane * CPL * 2;
        l += pw;
        if constexpr (CPL == 4) {
          const uint2 b = *reinterpret_cast<const uint2*>(vr);
          ov[0] = fmaf(pw, bf16_lo(b.x), ov[0]); ov[1] = fmaf(pw, bf16_hi(b.x), ov[1]);
          ov[2] = fmaf(pw, bf16_lo(b.y), ov[2]); ov[3] = fmaf(pw, bf16_hi(b.y), ov[3]);
        } else {
          const uint32_t b = *reinterpret_cast<const uint32_t*>(vr);
          ov[0] = fmaf(pw, bf16_lo(b), ov[0]); ov[1] = fmaf(pw, bf16_hi(b), ov[1]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(empty_bar + s));
    }
    // every warp used the same max: the merge is a plain sum
    consumer_sync();  // all score reads done before the buffer is reused
    float* wpart = sc;  // [kNW][D + 1]
#pragma unroll
    for (int i = 0; i < CPL; ++i) wpart[warp * (D + 1) + lane * CPL + i] = ov[i];
    if (lane == 0) wpart[warp * (D + 1) + D] = l;
    consumer_sync();
    for (int d = ctid; d < D + 2; d += kNW * 32) {
      float acc = 0.f;
      if (d != D) {
        const int dd = d == D + 1 ? D : d;
        for (int w = 0; w < kNW; ++w) acc += wpart[w * (D + 1) + dd];
      }
      part[d] = (d == D) ? m : acc;
    }
  } else {
    // ---- LUT of step t: LUT[c][g*J + j] = sum_w q_{j*W+w} * B^K_t[c][j][w]
    // The histogram later accumulates on top of these words (u32 adds wrap),
    // so the thread keeps the bits it wrote and subtracts them at the end.
    uint32_t lutb[kPer];
    {
      const int j = ctid % J;
      float qj[W];                 // q[j*W .. j*W+W) of this thread's slot j, log2 units
#pragma unroll
      for (int w = 0; w < W; ++w) qj[w] = load_q(p.q, p.q_bf16, unit * D + j * W + w) * p.scale_log2;
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const int c = (ctid + k * kNW * 32) / J;
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < W; ++w) acc = fmaf(qj[w], wk[k][w], acc);
        if (c >= p.C) acc = __int_as_float(0x7fc00000);  // NaN marks a code >= n_codes
        lutb[k] = __float_as_uint(acc);
#pragma unroll
        for (int g = 0; g < kCols / J; ++g) lut[c * kCols + g * J + j] = acc;
      }
    }
    const uint32_t lb = region | (uint32_t)(lane * 4);
    consumer_sync();

    // Each warp owns tiles warp + kNW*i (i < kTPW) of every chunk.  It copies
    // their code words (16 per lane) to registers and releases the stage at
    // once, so the producer refills it while the warp gathers.
    constexpr int kTPW = kTilesPerChunk / kNW;  // 2, 4, 8 for J = 32, 16, 8
    constexpr int kWPT = J / 4;                 // code words per tile and lane

    // ---- pass K: scores and split maximum
    float mx = -INFINITY;
    bool nan_seen = false;
    for (int k = 0; k < n_chunks_half; ++k) {
      const int s = k % kStages;
      if (!mbar_wait_bounded(smem_u32(full_bar + s), (k / kStages) & 1)) set_fault(p.status, LOOPVQ_FAULT_TIMEOUT);
      const uint8_t* st = stage_ptr(s);
      const int nt = min(kTilesPerChunk, n_tiles - k * kTilesPerChunk);
      uint32_t wd[kTPW][kWPT];
#pragma unroll
      for (int i = 0; i < kTPW; ++i) {
        if (warp + kNW * i < nt) {
          load_tile_words<J>(st + (warp + kNW * i) * 32 * J, lane, wd[i]);
        } else {
#pragma unroll
          for (int x = 0; x < kWPT; ++x) wd[i][x] = 0u;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(empty_bar + s));
#pragma unroll
      for (int i = 0; i < kTPW; i += 2) {
        const int tl = warp + kNW * i;
        if (tl < nt) {
          float sv[2];
          score_pair<J>(wd[i], wd[i + 1], lb, sv[0], sv[1]);
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int tok = (k * kTilesPerChunk + tl + kNW * u) * 32 + lane;
            const bool v = (tl + kNW * u < nt) && tok < n_tok;
            if (v && sv[u] != sv[u]) nan_seen = true;
            if (tl + kNW * u < nt) sc[tok] = v ? sv[u] : -INFINITY;
            mx = fmaxf(mx, v ? sv[u] : -INFINITY);
          }
        }
      }
    }
    if (nan_seen) set_fault(p.status, LOOPVQ_FAULT_CODE_RANGE);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) red[warp] = mx;
    consumer_sync();
    float m = -INFINITY;
    for (int w = 0; w < kNW; ++w) m = fmaxf(m, red[w]);
    // the table is done with: the region becomes the histogram (no zeroing:
    // every bin starts at the table word this thread wrote there)
    // fixed-point scale: n_tok * 2^S < 2^32 with S = clz(n_tok)
    const int S = __clz(max(n_tok, 1));
    const float scaleS = exp2f((float)S);

    // ---- pass V: weights into the histogram
    uint32_t qsum = 0;
    for (int k = n_chunks_half; k < n_chunks; ++k) {
      const int s = k % kStages;
      if (!mbar_wait_bounded(smem_u32(full_bar + s), (k / kStages) & 1)) set_fault(p.status, LOOPVQ_FAULT_TIMEOUT);
      const uint8_t* st = stage_ptr(s);
      const int kv = k - n_chunks_half;
      const int nt = min(kTilesPerChunk, n_tiles - kv * kTilesPerChunk);
      uint32_t wd[kTPW][kWPT];
#pragma unroll
      for (int i = 0; i < kTPW; ++i) {
        if (warp + kNW * i < nt) {
          load_tile_words<J>(st + (warp + kNW * i) * 32 * J, lane, wd[i]);
        } else {
#pragma unroll
          for (int x = 0; x < kWPT; ++x) wd[i][x] = 0u;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(empty_bar + s));
#pragma unroll
      for (int i = 0; i < kTPW; i += 2) {
        const int tl = warp + kNW * i;
        if (tl < nt) {
          uint32_t qv[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int tok = (kv * kTilesPerChunk + tl + kNW * u) * 32 + lane;
            qv[u] = 0;
            if (tl + kNW * u < nt && tok < n_tok) {
              const float pw = exp2f(sc[tok] - m);
              const uint32_t seq = (uint32_t)(body_off + tok0 + tok);
              const float uu = (float)((seq * 2654435769u) >> 8) * (1.0f / 16777216.0f);
              qv[u] = __float2uint_rd(fmaf(pw, scaleS, uu));
            }
            qsum += qv[u];
          }
          hist_pair<J>(wd[i], wd[i + 1], lb, qv[0], qv[1]);
        }
      }
    }
    // the value codebook slice (code-major entries (c, j) = ctid + 512k),
    // which the producer bulk-copied into the drained ring stages
    const int n_slice = (n_tok == 0) ? 0 : (int)((p.C * D * sizeof(CBT) + kStageBytes - 1) / kStageBytes);
    for (int i = 0; i < n_slice; ++i) {
      const int k = n_chunks + i;
      if (!mbar_wait_bounded(smem_u32(full_bar + (k % kStages)), (k / kStages) & 1))
        set_fault(p.status, LOOPVQ_FAULT_TIMEOUT);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) qsum += __shfl_xor_sync(0xffffffffu, qsum, o);
    if (lane == 0) reinterpret_cast<uint32_t*>(red)[kNW + warp] = qsum;
    consumer_sync();

    // ---- epilogue: o[d] = 2^-S sum_c hist[j][c] B^V_t[c][j][w].  Thread
    // ctid accumulates its W outputs over entries (c, j) = ctid + 512k; the
    // 512/J partial groups per output are summed through shared memory (the
    // score buffer is free by now).
    {
      const int j = ctid % J;
      float hf[kPer];
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const int c = (ctid + k * kNW * 32) / J;
        uint32_t hs = 0;
#pragma unroll
        for (int g = 0; g < kCols / J; ++g) hs += hist[c * kCols + g * J + j];
        hs -= (uint32_t)(kCols / J) * lutb[k];
        hf[k] = c < p.C ? (float)hs : 0.f;
      }
      float acc[W];
#pragma unroll
      for (int w = 0; w < W; ++w) acc[w] = 0.f;
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const int e = ctid + k * kNW * 32;
        const uint32_t off = (uint32_t)e * W * sizeof(CBT);
        const CBT* src = reinterpret_cast<const CBT*>(stage_ptr((n_chunks + (int)(off / kStageBytes)) % kStages) +
                                                      off % kStageBytes);
        float vv[W];
        load_vec<W>(src, n_slice > 0 && e / J < p.C, vv);
#pragma unroll
        for (int w = 0; w < W; ++w) acc[w] = fmaf(hf[k], vv[w], acc[w]);
      }
      // bins of codes >= n_codes must be empty
      if (p.C < 256) {
        bool any = false;
        for (int e = p.C * kCols + ctid; e < 256 * kCols; e += kNW * 32) any |= hist[e] != 0x7fc00000u;
        if (any) set_fault(p.status, LOOPVQ_FAULT_CODE_RANGE);
      }
      // lanes l and l + J of a warp hold the same slot: fold them first
#pragma unroll
      for (int o = J; o < 32; o <<= 1) {
#pragma unroll
        for (int w = 0; w < W; ++w) acc[w] += __shfl_xor_sync(0xffffffffu, acc[w], o);
      }
      float* ored = sc;  // [kNW][D] per-warp partial sums; scores are no longer read
      if (lane < J) {
        if constexpr (W % 4 == 0) {
#pragma unroll
          for (int w = 0; w < W; w += 4)
            *reinterpret_cast<float4*>(ored + warp * D + j * W + w) = make_float4(acc[w], acc[w + 1], acc[w + 2], acc[w + 3]);
        } else {
#pragma unroll
          for (int w = 0; w < W; ++w) ored[warp * D + j * W + w] = acc[w];
        }
      }
      consumer_sync();
      if (ctid < D) {
        float o = 0.f;
#pragma unroll
        for (int i = 0; i < kNW; ++i) o += ored[i * D + ctid];
        part[ctid] = o * (1.f / scaleS);  // exact: a power of two
      }
    }
    if (ctid == 0) {
      uint64_t tot = 0;
      for (int w = 0; w < kNW; ++w) tot += reinterpret_cast<uint32_t*>(red)[kNW + w];
      part[D] = m;
      part[D + 1] = (float)tot * (1.f / scaleS);
    }
  }

  // the merge kernel, launched right after as a dependent, combines the splits
}

// Merge of the splits of every (request, query head): one CTA of D threads
// per unit, launched as a programmatic dependent of the decode kernel (it
// starts while the decode runs and waits for its completion before reading
// the partials).  Thread d loads column d of up to 32 partial rows at once and
// lane s of every warp the (m, l) of split s -- one round trip to L2, no
// shared memory -- and the log-sum-exp weights travel by shuffles; more than
// 32 splits merge online, 32 at a time.
constexpr int kMergeChunk = 32;

template <int D>
__global__ void __launch_bounds__(D) merge_kernel(const DecodeParams p) {
  griddep_launch_dependents();
  const int tid = threadIdx.x, lane = tid & 31;
  const int hq = blockIdx.x, r = blockIdx.y;
  const size_t unit = ((size_t)blockIdx.z * p.batch + r) * p.Hq + hq;  // z: step of a multi-step launch
  int ctx = __ldg(p.ctx_len + r);
  if (ctx < 0 || ctx > p.max_ctx) ctx = 0;  // reported by the decode kernel
  const CtxSplit cs = ctx_split(ctx, p.n_sink, p.n_recent, p.page);
  const int n_win = cs.sink + cs.recent;
  const int n_splits = ctx == 0 ? 0 : (n_win > 0 ? 1 : 0) + (cs.body + p.split_len - 1) / p.split_len;
  griddep_wait();
  const float* part = p.partials + unit * p.max_splits * (size_t)(D + 4);
  float M = -INFINITY, Ls = 0.f, o = 0.f;  // running merge
  for (int c0 = 0; c0 < n_splits; c0 += kMergeChunk) {
    const int nc = min(kMergeChunk, n_splits - c0);
    const float* rows = part + (size_t)c0 * (D + 4);
    float ov[kMergeChunk];
#pragma unroll
    for (int s = 0; s < kMergeChunk; ++s) ov[s] = s < nc ? __ldcg(rows + (size_t)s * (D + 4) + tid) : 0.f;
    const float ms = lane < nc ? __ldcg(rows + (size_t)lane * (D + 4) + D) : -INFINITY;
    const float ls = lane < nc ? __ldcg(rows + (size_t)lane * (D + 4) + D + 1) : 0.f;
    float Mc = ms;
#pragma unroll
    for (int x = 16; x >= 1; x >>= 1) Mc = fmaxf(Mc, __shfl_xor_sync(0xffffffffu, Mc, x));
    const float Mn = fmaxf(M, Mc);
    const float e = ms == -INFINITY ? 0.f : exp2f(ms - Mn);
    float Lc = ls * e;
#pragma unroll
    for (int x = 16; x >= 1; x >>= 1) Lc += __shfl_xor_sync(0xffffffffu, Lc, x);
    const float keep = M == -INFINITY ? 0.f : exp2f(M - Mn);
    float oc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int s = 0; s < kMergeChunk; ++s) oc[s & 3] = fmaf(ov[s], __shfl_sync(0xffffffffu, e, s), oc[s & 3]);
    o = fmaf(o, keep, (oc[0] + oc[1]) + (oc[2] + oc[3]));
    Ls = fmaf(Ls, keep, Lc);
    M = Mn;
  }
  const bool ok = M != -INFINITY && Ls > 0.f;
  const float res = ok ? o * __frcp_rn(Ls) : 0.f;
  if (p.out_bf16)
    reinterpret_cast<__nv_bfloat16*>(p.out)[unit * D + tid] = __float2bfloat16_rn(res);
  else
    reinterpret_cast<float*>(p.out)[unit * D + tid] = res;
  if (p.lse && tid == 0) p.lse[unit] = ok ? (M + log2f(Ls)) * 0.6931471805599453f : -INFINITY;
}

// Launches the decode kernel as a programmatic dependent of the previous
// kernel in the stream (it may start while that kernel finishes; the kernel
// waits for it before touching anything it may write).
static cudaError_t launch_pdl(const void* fn, dim3 grid, cudaStream_t s, DecodeParams* p,
                              unsigned threads = kThreads, size_t smem = kDynSmem) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  void* args[] = {p};
  return cudaLaunchKernelExC(&cfg, fn, args);
}

// Host-side plan: body tokens per split so that the grid fills the SMs.
struct DecodePlan {
  int n_body_splits, split_len, max_splits;
};
inline DecodePlan decode_plan(int64_t units, int max_body, int n_sm, int cap = kSplitCap) {
  DecodePlan pl;
  int need = (max_body + cap - 1) / cap;  // score buffer and fixed-point bound
  int fill = (int)(n_sm / (units > 0 ? units : 1)) - 1;  // one window split per unit
  int cap_by_tiles = (max_body + 255) / 256;             // >= 256 tokens per split
  int s = need;
  if (fill > s) s = fill < cap_by_tiles ? fill : cap_by_tiles;
  if (s < 1) s = 1;
  int len = (max_body + s - 1) / s;
  len = ((len + 31) / 32) * 32;
  if (len < 32) len = 32;
  if (len > cap) len = cap;
  pl.split_len = len;
  pl.n_body_splits = max_body > 0 ? (max_body + len - 1) / len : 0;
  pl.max_splits = pl.n_body_splits + 1;
  return pl;
}

static int max_body_tokens(const loopvq_cache_layout* L) {
  return ctx_split(L->max_ctx_len, L->n_sink, L->n_recent, L->page).body;
}

// workspace bound independent of the device: plan with a generous SM count
static WsLayout decode_ws(const Geo& g, const loopvq_cache_layout* L, int n_steps = 1) {
  const int64_t units = (int64_t)L->batch * g.Hq * n_steps;
  const int cap = long_splits(g.D, (int)cb_elem_bytes(g)) ? kSplitCapLong : kSplitCap;
  DecodePlan pl = decode_plan(units, max_body_tokens(L), 1024, cap);
  return ws_layout(units, pl.max_splits, g.D);
}

static loopvq_status check_layout(const loopvq_cache_layout* L) {
  if (!L || L->batch < 1 || L->n_sink < 0 || L->n_recent < 0 || L->page < 1 || L->max_ctx_len < 0)
    return LOOPVQ_ERR_INVALID_ARG;
  const bool paged = L->flags & LOOPVQ_LAYOUT_PAGED_BODY, ring = L->flags & LOOPVQ_LAYOUT_RING_WINDOW;
  if (L->flags & ~(LOOPVQ_LAYOUT_STATIC_INPUTS | LOOPVQ_LAYOUT_PAGED_BODY | LOOPVQ_LAYOUT_RING_WINDOW))
    return LOOPVQ_ERR_INVALID_ARG;
  if (!L->ctx_len || !L->win_off || (!paged && !L->body_off)) return LOOPVQ_ERR_INVALID_ARG;
  if (L->body_pool_tokens < 0 || (L->body_pool_tokens & 31) || L->win_pool_tokens < 0) return LOOPVQ_ERR_INVALID_ARG;
  if (paged) {
    if (!L->body_pages || L->body_page_tokens < 32 || (L->body_page_tokens & 31) ||
        L->body_page_tokens % L->page || L->max_body_pages < 1)
      return LOOPVQ_ERR_INVALID_ARG;
    const int64_t body = ctx_split(L->max_ctx_len, L->n_sink, L->n_recent, L->page).body;
    if ((int64_t)L->max_body_pages * L->body_page_tokens < body) return LOOPVQ_ERR_INVALID_ARG;
  }
  if (ring && (!L->win_head || L->win_ring < 1 || L->win_ring < L->n_recent + L->page - 1))
    return LOOPVQ_ERR_INVALID_ARG;
  if ((L->new_k == nullptr) != (L->new_v == nullptr)) return LOOPVQ_ERR_INVALID_ARG;
  if (((uintptr_t)L->new_k & 3) || ((uintptr_t)L->new_v & 3)) return LOOPVQ_ERR_INVALID_ARG;
  return LOOPVQ_OK;
}

// Layout fields of the kernel parameters shared by both entry points.
static void fill_layout_params(DecodeParams& p, const loopvq_cache_layout* L) {
  p.paged = (L->flags & LOOPVQ_LAYOUT_PAGED_BODY) ? 1 : 0;
  p.body_pages = L->body_pages;
  p.body_page_tokens = p.paged ? L->body_page_tokens : 32;
  p.max_body_pages = L->max_body_pages;
  p.ring = (L->flags & LOOPVQ_LAYOUT_RING_WINDOW) ? 1 : 0;
  p.win_head = L->win_head;
  p.win_ring = p.ring ? L->win_ring : 1;
  p.new_k = (const __nv_bfloat16*)L->new_k;
  p.new_v = (const __nv_bfloat16*)L->new_v;
}

}  // namespace loopvq

using namespace loopvq;

namespace loopvq {

// Checks the arguments shared by the decode entry points and fills the kernel
// parameters for steps first_step .. first_step + n_steps - 1 (all but the
// workspace pointers).
static loopvq_status decode_setup(const loopvq_codebook_desc* desc, const void* cbK_packed, const void* cbV_packed,
                                  const loopvq_cache_layout* layout, const uint8_t* idxK_pool,
                                  const uint8_t* idxV_pool, const void* winK, const void* winV, const void* q,
                                  loopvq_dtype q_dtype, int32_t first_step, int32_t n_steps, float softmax_scale,
                                  void* out, loopvq_dtype out_dtype, float* lse_out, Geo* g_out,
                                  DecodeParams* p_out) {
  Geo g;
  loopvq_status st = make_geo(desc, &g);
  if (st != LOOPVQ_OK) return st;
  if ((st = check_layout(layout)) != LOOPVQ_OK) return st;
  if (g.J != 8 && g.J != 16 && g.J != 32) return LOOPVQ_ERR_UNSUPPORTED;
  if (g.D != 64 && g.D != 128) return LOOPVQ_ERR_UNSUPPORTED;
  if (n_steps < 1 || first_step < 0 || first_step > g.T - n_steps) return LOOPVQ_ERR_INVALID_ARG;
  if (q_dtype != LOOPVQ_F32 && q_dtype != LOOPVQ_BF16) return LOOPVQ_ERR_INVALID_ARG;
  if (out_dtype != LOOPVQ_F32 && out_dtype != LOOPVQ_BF16) return LOOPVQ_ERR_INVALID_ARG;
  if (!(softmax_scale == softmax_scale)) return LOOPVQ_ERR_INVALID_ARG;
  if (!cbK_packed || !cbV_packed || !idxK_pool || !idxV_pool || !winK || !winV || !q || !out)
    return LOOPVQ_ERR_INVALID_ARG;
  if (((uintptr_t)idxK_pool & 15) || ((uintptr_t)idxV_pool & 15) || ((uintptr_t)winK & 15) ||
      ((uintptr_t)winV & 15) || ((uintptr_t)cbK_packed & 15) || ((uintptr_t)cbV_packed & 15))
    return LOOPVQ_ERR_INVALID_ARG;
  const int64_t units = (int64_t)layout->batch * g.Hq * n_steps;
  const int cap = long_splits(g.D, (int)cb_elem_bytes(g)) ? kSplitCapLong : kSplitCap;
  const DecodePlan pl = decode_plan(units, max_body_tokens(layout), device_sm_count(), cap);
  if (units > 65535LL * 65535LL || pl.max_splits > kMaxCombineSplits || layout->batch > 65535 ||
      (int64_t)g.Hq * n_steps > 65535)
    return LOOPVQ_ERR_UNSUPPORTED;

  DecodeParams& p = *p_out;
  p.T = g.T; p.Tc = g.Tc; p.H = g.H; p.Hq = g.Hq; p.D = g.D; p.J = g.J; p.W = g.W; p.C = g.C;
  p.loop_step = first_step;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.batch = layout->batch; p.n_sink = layout->n_sink; p.n_recent = layout->n_recent;
  p.page = layout->page; p.max_ctx = layout->max_ctx_len;
  p.ctx_len = layout->ctx_len; p.body_off = layout->body_off; p.win_off = layout->win_off;
  p.body_pool_tokens = layout->body_pool_tokens; p.win_pool_tokens = layout->win_pool_tokens;
  const size_t eb = cb_elem_bytes(g);
  const size_t step_off = packed_slices_offset_bytes(g) + (size_t)first_step * slice_elems_per_step(g) * eb;
  p.cbK_slice = (const uint8_t*)cbK_packed + step_off;
  p.cbV_slice = (const uint8_t*)cbV_packed + step_off;
  const size_t blk_bytes = (size_t)g.H * layout->body_pool_tokens * g.J;
  p.idxK = idxK_pool + (first_step / g.Tc) * blk_bytes;
  p.idxV = idxV_pool + (first_step / g.Tc) * blk_bytes;
  const size_t win_step = (size_t)g.H * layout->win_pool_tokens * g.D;
  p.winK = (const __nv_bfloat16*)winK + first_step * win_step;
  p.winV = (const __nv_bfloat16*)winV + first_step * win_step;
  p.q = q; p.q_bf16 = q_dtype == LOOPVQ_BF16;
  p.out = out; p.out_bf16 = out_dtype == LOOPVQ_BF16; p.lse = lse_out;
  p.n_steps = n_steps;
  p.slice_step_elems = (int64_t)slice_elems_per_step(g);
  p.win_step_elems = (int64_t)win_step;
  p.idx_blk_bytes = (int64_t)blk_bytes;
  p.split_len = pl.split_len;
  p.max_splits = pl.max_splits;
  p.static_inputs = (layout->flags & LOOPVQ_LAYOUT_STATIC_INPUTS) ? 1 : 0;
  fill_layout_params(p, layout);
  *g_out = g;
  return LOOPVQ_OK;
}

// The split kernel and its dependent merge kernel on `s`.
static loopvq_status decode_launch(const Geo& g, DecodeParams& p, cudaStream_t s) {
  const dim3 grid(g.Hq * p.n_steps, p.max_splits, p.batch);
  const dim3 mgrid(g.Hq, p.batch, p.n_steps);
#define LOOPVQ_LAUNCH(JJ, DD, CBT)                                                                    \
  do {                                                                                               \
    auto kfn = p.n_steps > 1 ? decode_kernel<JJ, DD, CBT, true> : decode_kernel<JJ, DD, CBT, false>; \
    if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, kDynSmem) != cudaSuccess) \
      return LOOPVQ_ERR_CUDA;                                                                        \
    if (launch_pdl((const void*)kfn, grid, s, &p) != cudaSuccess) return LOOPVQ_ERR_CUDA;           \
    if (launch_pdl((const void*)merge_kernel<DD>, mgrid, s, &p, DD, 0) != cudaSuccess)               \
      return LOOPVQ_ERR_CUDA;                                                                        \
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

static loopvq_status decode_with_workspace(const loopvq_codebook_desc* desc, const void* cbK_packed,
                                           const void* cbV_packed, const loopvq_cache_layout* layout,
                                           const uint8_t* idxK_pool, const uint8_t* idxV_pool, const void* winK,
                                           const void* winV, const void* q, loopvq_dtype q_dtype,
                                           int32_t first_step, int32_t n_steps, float softmax_scale, void* out,
                                           loopvq_dtype out_dtype, float* lse_out, void* workspace,
                                           size_t workspace_bytes, loopvq_stream_t stream) {
  Geo g;
  DecodeParams p;
  loopvq_status st = decode_setup(desc, cbK_packed, cbV_packed, layout, idxK_pool, idxV_pool, winK, winV, q,
                                  q_dtype, first_step, n_steps, softmax_scale, out, out_dtype, lse_out, &g, &p);
  if (st != LOOPVQ_OK) return st;
  if (!workspace || ((uintptr_t)workspace & 255)) return LOOPVQ_ERR_INVALID_ARG;
  const WsLayout ws = decode_ws(g, layout, n_steps);
  if (workspace_bytes < ws.total) return LOOPVQ_ERR_WORKSPACE_TOO_SMALL;
  p.status = (uint32_t*)workspace;
  p.partials = (float*)((uint8_t*)workspace + ws.partials_off);
  return decode_launch(g, p, (cudaStream_t)stream);
}

}  // namespace loopvq

extern "C" size_t loopvq_decode_workspace_bytes(const loopvq_codebook_desc* desc,
                                                const loopvq_cache_layout* layout) {
  return loopvq_decode_steps_workspace_bytes(desc, layout, 1);
}

extern "C" size_t loopvq_decode_steps_workspace_bytes(const loopvq_codebook_desc* desc,
                                                      const loopvq_cache_layout* layout, int32_t n_steps) {
  Geo g;
  if (make_geo(desc, &g) != LOOPVQ_OK || check_layout(layout) != LOOPVQ_OK || n_steps < 1 || n_steps > g.T) return 0;
  return decode_ws(g, layout, n_steps).total;
}

extern "C" loopvq_status loopvq_decode_attn(const loopvq_codebook_desc* desc, const void* cbK_packed,
                                            const void* cbV_packed, const loopvq_cache_layout* layout,
                                            const uint8_t* idxK_pool, const uint8_t* idxV_pool,
                                            const void* winK, const void* winV, const void* q,
                                            loopvq_dtype q_dtype, int32_t loop_step, float softmax_scale,
                                            void* out, loopvq_dtype out_dtype, float* lse_out,
                                            void* workspace, size_t workspace_bytes,
                                            loopvq_stream_t stream) {
  return decode_with_workspace(desc, cbK_packed, cbV_packed, layout, idxK_pool, idxV_pool, winK, winV, q, q_dtype,
                               loop_step, 1, softmax_scale, out, out_dtype, lse_out, workspace, workspace_bytes,
                               stream);
}

extern "C" loopvq_status loopvq_decode_attn_steps(const loopvq_codebook_desc* desc, const void* cbK_packed,
                                                  const void* cbV_packed, const loopvq_cache_layout* layout,
                                                  const uint8_t* idxK_pool, const uint8_t* idxV_pool,
                                                  const void* winK, const void* winV, const void* q,
                                                  loopvq_dtype q_dtype, int32_t first_step, int32_t n_steps,
                                                  float softmax_scale, void* out, loopvq_dtype out_dtype,
                                                  float* lse_out, void* workspace, size_t workspace_bytes,
                                                  loopvq_stream_t stream) {
  return decode_with_workspace(desc, cbK_packed, cbV_packed, layout, idxK_pool, idxV_pool, winK, winV, q, q_dtype,
                               first_step, n_steps, softmax_scale, out, out_dtype, lse_out, workspace,
                               workspace_bytes, stream);
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
  DecodeParams p;
  loopvq_status st = decode_setup(desc, cbK_packed, cbV_packed, layout, idxK_pool, idxV_pool, winK, winV, q,
                                  q_dtype, loop_step, 1, softmax_scale, out, out_dtype, lse_out, &g, &p);
  if (st != LOOPVQ_OK) return st;
  if ((uintptr_t)fault_bits & 3) return LOOPVQ_ERR_INVALID_ARG;
  const WsLayout ws = decode_ws(g, layout);
  if (ws.total > kLoopvqStaticScratchBytes) return LOOPVQ_ERR_WORKSPACE_TOO_SMALL;

  void* scratch = nullptr;
  if ((st = static_scratch(&scratch)) != LOOPVQ_OK) return st;
  // every split writes its partial before the merge kernel reads it, so
  // nothing in the array needs clearing; faults go to the caller's word (or
  // nowhere when fault_bits is null)
  p.status = fault_bits;
  p.partials = (float*)((uint8_t*)scratch + ws.partials_off);
  return decode_launch(g, p, (cudaStream_t)stream);
}
