// decode_attn.cuh -- paged decode attention (one query token per sequence).
//
// Method: Q.K^T, online softmax (running max / running sum) and P.V in one
// pass over the K/V pages of a sequence, found through its block table
// ("从零构建CUDA推理引擎：Tiny-Infer项目的技术深度解析", sections
// "Flash Attention：内存与计算的重平衡" and "分页KV缓存：借鉴操作系统的内存管理";
// "5 Fun Projects for LLM Inference Engineering", section 2).  Decode is bound
// by reading the KV cache from HBM ("Triton融合算子优化：LLM推理性能提升3倍的
// 工程实践", section 一), so this kernel is built around the copy engine, not
// the tensor cores.
//
// B200 design:
//   * Work is cut into segments: (sequence b, a group of HG query heads that
//     share one kv head).  The HG query rows live in registers, so every K/V
//     byte is read from HBM once per group (grouped-query reuse).
//   * Pages move by 1-D bulk copies (cp.async.bulk) of whole pages -- a
//     (block, kv head) page is one contiguous 4 KB (D=128) or 2 KB (D=64) run
//     -- into each warp's own SW-stage shared-memory ring, completion tracked
//     by one mbarrier per stage.  Each consumer warp has a producer warp
//     that issues its copies and refills a stage when the consumer hands it
//     back, so copy issue never interrupts the arithmetic (it matters most at
//     D=64, with twice the copies per byte); a register split (setmaxnreg)
//     keeps two such CTAs per SM.  (Without producers -- PROD = false -- each
//     warp's lane 0 refills its own stages between compute steps.)
//   * Two CTAs per SM (shared-memory carveout at its maximum) keep
//     2 x NW x SW stages -- 192 KB -- in flight per SM, which is what
//     Little's law asks for at full HBM bandwidth.
//   * A key row is split over LPR = D/16 lanes (16 elements, two 16-byte
//     vectors each), so a warp covers 32/LPR rows per instruction and a dot
//     product needs only log2(LPR) shuffle steps.  Products and P.V updates
//     use packed fp32 (FFMA2) on element pairs.  Each lane keeps its own
//     running max, sum and fp32 accumulator; lanes and warps merge by
//     log-sum-exp when a segment (or a CTA's share of it) is done.
//   * Shared-memory reads are conflict-free: for D=128 the 8 lanes of a row
//     read 128 contiguous bytes per phase; for D=64 odd row groups read their
//     two vectors in swapped order, and their q / accumulator registers are
//     kept in that swapped order too.
//   * One CTA per (segment, split of pages_per_split pages).  With one split
//     the CTA writes the bf16 output itself; with several, each split writes
//     a normalised fp32 partial and its log2-sum-exp, and lse_merge_kernel
//     combines them.  The block scheduler hands CTAs to SMs as others finish,
//     which absorbs ragged lengths and SMs that stream at different rates.
#pragma once
#include "pkv_common.cuh"

namespace pkv {

constexpr int kPageRows = 16;  // block_size supported by the attention kernels

struct DecodeParams {
  __nv_bfloat16* out;            // [B][Hq][D]
  float* o_part;                 // split partials [B][Hq][C][D]
  float* lse_part;               // their log2-sum-exp [B][Hq][C]
  const __nv_bfloat16* q;        // [B][Hq][D]
  const unsigned char* k_cache;  // [NB][Hkv][16][D] bf16 (int8 codes for the int8 cache)
  const unsigned char* v_cache;
  const float* k_scale;          // int8 cache: [NB][Hkv][16] fp32 scale per row
  const float* v_scale;
  const int32_t* block_tables;   // [B][MB]
  const int32_t* context_lens;   // [B]
  int32_t B, Hq, Hkv, NB, MB;
  int32_t G;                     // Hq / Hkv
  int32_t nsub;                  // G / HG head groups per kv head
  int32_t pages_per_split;
  int32_t num_splits;            // 1: write bf16 output directly
  int32_t cap_tokens;            // longest context this launch can hold
  int32_t window;                // > 0: the query sees only its last `window` keys
  float scale_log2;              // scale * log2(e)
};

// First key a decode query (position L - 1) sees: 0, or L - window under a
// sliding window of `window` keys (a query at p sees keys p - window < j <= p).
__device__ __forceinline__ int window_first_key(int L, int window) {
  return (window > 0 && L > window) ? L - window : 0;
}

// A ring stage holds PPS consecutive pages of one sequence: their K pages
// side by side (ROWS = 16 * PPS contiguous key rows), then their V pages.
// PROD: each of the NW consumer warps has a producer warp that issues its
// copies (NW more warps, and an "empty" barrier per stage).
template <int D, int HG, int NW, int SW, int PPS, bool PROD = false>
struct DecodeShape {
  static_assert(D == 64 || D == 128, "head_dim");
  static constexpr int LPR = D / 16;              // lanes sharing one key row
  static constexpr int RPW = 32 / LPR;            // rows per warp step
  static constexpr int ROWS = kPageRows * PPS;    // key rows per stage
  static constexpr int TPL = ROWS / RPW;          // rows per lane per stage
  static constexpr int PAGE_BYTES = kPageRows * D * 2;
  static constexpr int STAGE_BYTES = 2 * PPS * PAGE_BYTES;
  static constexpr int THREADS = NW * 32 * (PROD ? 2 : 1);
  // register split of the producer form: consumers (warpgroup 0) up to
  // REGS_CONS, producers (warpgroup 1) down to REGS_PROD, within the 128 per
  // thread that two CTAs of THREADS threads leave each on an SM
  static constexpr int REGS_CONS = 216, REGS_PROD = 40, REGS_LAUNCH = 128;
  static_assert(!PROD || (NW == 4 && REGS_CONS + REGS_PROD <= 2 * REGS_LAUNCH), "producer register split");
  static constexpr int WARP_RING = SW * STAGE_BYTES;
  static constexpr int RING_BYTES = NW * WARP_RING;
  // one warp's merge data: acc [HG][D], m [HG], l [HG]; stride kept 16-byte aligned
  static constexpr int MERGE_STRIDE = (HG * D + 2 * HG + 3) / 4 * 4;
  static_assert(MERGE_STRIDE * 4 <= WARP_RING, "merge data must fit the warp's ring");
  // rings, then "full" barriers, then (PROD) "empty" barriers; merge data
  // reuses each warp's ring
  static constexpr int BAR_OFFSET = RING_BYTES;
  static constexpr int EMPTY_OFFSET = BAR_OFFSET + NW * SW * 8;
  static constexpr int SMEM_BYTES = EMPTY_OFFSET + (PROD ? NW * SW * 8 : 0);
};

__device__ __forceinline__ float2 widen2(uint32_t w) {
  return make_float2(bf16lo_to_f32(w), bf16hi_to_f32(w));
}

// Per-lane running softmax state for HG query heads over the lane's 16
// elements of D: running max m, running sum l, fp32 accumulator (8 pairs).
template <int HG>
struct LaneState {
  float m[HG], l[HG];
  float2 acc[HG][8];
  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int h = 0; h < HG; ++h) {
      m[h] = -INFINITY;
      l[h] = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[h][e] = make_float2(0.f, 0.f);
    }
  }
};

// The lane's 16 q elements of each of the HG heads, as 8 pairs, pre-scaled.
template <int D, int HG>
__device__ __forceinline__ void load_q(float2 (&q2)[HG][8], const __nv_bfloat16* q_row0, int ch0,
                                       int ch1, float scale_log2) {
#pragma unroll
  for (int h = 0; h < HG; ++h) {
    const uint4* qrow = reinterpret_cast<const uint4*>(q_row0 + (size_t)h * D);
    const uint4 a = __ldg(qrow + ch0), c = __ldg(qrow + ch1);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
    const float2 sc2 = make_float2(scale_log2, scale_log2);
#pragma unroll
    for (int e = 0; e < 8; ++e) q2[h][e] = __fmul2_rn(widen2(w[e]), sc2);
  }
}

// ROWS key rows (K at kp, V at vp, row stride D) into the lane state.  Rows
// outside [nstart, nvalid) -- past the end of the sequence or of the copied
// pages, or before a sliding window -- take no part in the max and are never
// read from V.
template <int D, int HG, int ROWS>
__device__ __forceinline__ void attend_rows(LaneState<HG>& st, const float2 (&q2)[HG][8],
                                            const unsigned char* kp, const unsigned char* vp,
                                            int nstart, int nvalid, int rg, int ch0, int ch1) {
  constexpr int LPR = D / 16, RPW = 32 / LPR, TPL = ROWS / RPW;
  float sc[TPL][HG];
#pragma unroll
  for (int t = 0; t < TPL; ++t) {
    const int r = rg + t * RPW;
    const uint4* krow = reinterpret_cast<const uint4*>(kp + r * D * 2);
    const uint4 ka = krow[ch0], kb = krow[ch1];
    const float2 k2[8] = {widen2(ka.x), widen2(ka.y), widen2(ka.z), widen2(ka.w),
                          widen2(kb.x), widen2(kb.y), widen2(kb.z), widen2(kb.w)};
#pragma unroll
    for (int h = 0; h < HG; ++h) {
      float2 d = __fmul2_rn(q2[h][0], k2[0]);
#pragma unroll
      for (int e = 1; e < 8; ++e) d = __ffma2_rn(q2[h][e], k2[e], d);
      sc[t][h] = d.x + d.y;
    }
  }
#pragma unroll
  for (int off = LPR / 2; off >= 1; off >>= 1)
#pragma unroll
    for (int t = 0; t < TPL; ++t)
#pragma unroll
      for (int h = 0; h < HG; ++h) sc[t][h] += __shfl_xor_sync(0xffffffffu, sc[t][h], off);

  bool valid[TPL];
#pragma unroll
  for (int t = 0; t < TPL; ++t) valid[t] = rg + t * RPW < nvalid && rg + t * RPW >= nstart;

  float mp[HG];
  bool grow = false;
#pragma unroll
  for (int h = 0; h < HG; ++h) {
    mp[h] = -INFINITY;
#pragma unroll
    for (int t = 0; t < TPL; ++t)
      if (valid[t]) mp[h] = fmaxf(mp[h], sc[t][h]);
    grow |= mp[h] > st.m[h];
  }
  if (__any_sync(0xffffffffu, grow)) {
#pragma unroll
    for (int h = 0; h < HG; ++h) {
      const float mn = fmaxf(st.m[h], mp[h]);
      const float alpha = (mn == -INFINITY) ? 1.f : ex2(st.m[h] - mn);
      st.m[h] = mn;
      st.l[h] *= alpha;
      const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
      for (int e = 0; e < 8; ++e) st.acc[h][e] = __fmul2_rn(st.acc[h][e], a2);
    }
  }
#pragma unroll
  for (int t = 0; t < TPL; ++t) {
    if (!valid[t]) continue;  // canary / stale rows are never touched
    const int r = rg + t * RPW;
    const uint4* vrow = reinterpret_cast<const uint4*>(vp + r * D * 2);
    const uint4 va = vrow[ch0], vb = vrow[ch1];
    const float2 v2[8] = {widen2(va.x), widen2(va.y), widen2(va.z), widen2(va.w),
                          widen2(vb.x), widen2(vb.y), widen2(vb.z), widen2(vb.w)};
#pragma unroll
    for (int h = 0; h < HG; ++h) {
      const float pr = ex2(sc[t][h] - st.m[h]);
      st.l[h] += pr;
      const float2 pp = make_float2(pr, pr);
#pragma unroll
      for (int e = 0; e < 8; ++e) st.acc[h][e] = __ffma2_rn(pp, v2[e], st.acc[h][e]);
    }
  }
}

// Four int8 codes (one 32-bit word) to four exact floats: a code c becomes
// (2^23 + (c + 128)) - (2^23 + 128); a byte permute builds the first term's
// bit pattern, one packed subtract finishes.
__device__ __forceinline__ void widen_i8x4(uint32_t w, float2& lo, float2& hi) {
  const uint32_t x = w ^ 0x80808080u;  // biased codes c + 128
  const float2 bias = make_float2(-8388736.f, -8388736.f);
  lo = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(x, 0x4B000000u, 0x7540)),
                              __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7541))), bias);
  hi = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(x, 0x4B000000u, 0x7542)),
                              __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7543))), bias);
}

// Merge the row groups of a warp (lanes holding the same D-slice) by
// log-sum-exp; afterwards lanes 0..LPR-1 hold the warp's result in natural
// element order.
template <int D, int HG, bool SWAPPED = (D == 64)>
__device__ __forceinline__ void warp_merge(LaneState<HG>& st) {
  constexpr int LPR = D / 16;
#pragma unroll
  for (int off = LPR; off < 32; off <<= 1) {
    const int flip = (SWAPPED && off == LPR) ? 4 : 0;  // partner keeps the other order
#pragma unroll
    for (int h = 0; h < HG; ++h) {
      const float mo = __shfl_xor_sync(0xffffffffu, st.m[h], off);
      const float lo = __shfl_xor_sync(0xffffffffu, st.l[h], off);
      const float mn = fmaxf(st.m[h], mo);
      const float a = (mn == -INFINITY) ? 0.f : ex2(st.m[h] - mn);
      const float c = (mn == -INFINITY) ? 0.f : ex2(mo - mn);
      float2 recv[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        recv[e].x = __shfl_xor_sync(0xffffffffu, st.acc[h][e ^ flip].x, off);
        recv[e].y = __shfl_xor_sync(0xffffffffu, st.acc[h][e ^ flip].y, off);
      }
      const float2 a2 = make_float2(a, a), c2 = make_float2(c, c);
#pragma unroll
      for (int e = 0; e < 8; ++e) st.acc[h][e] = __ffma2_rn(st.acc[h][e], a2, __fmul2_rn(recv[e], c2));
      st.l[h] = st.l[h] * a + lo * c;
      st.m[h] = mn;
    }
  }
}

// Lanes 0..LPR-1 of a warp write its merged state to `mine` ([HG][D] acc,
// [HG] m, [HG] l; 16-byte aligned).
template <int D, int HG>
__device__ __forceinline__ void warp_store(float* mine, const LaneState<HG>& st, int rg, int sub, int ch0,
                                           int ch1) {
  if (rg != 0) return;
#pragma unroll
  for (int h = 0; h < HG; ++h) {
    float4* dst = reinterpret_cast<float4*>(mine + h * D);
    dst[2 * ch0] = make_float4(st.acc[h][0].x, st.acc[h][0].y, st.acc[h][1].x, st.acc[h][1].y);
    dst[2 * ch0 + 1] = make_float4(st.acc[h][2].x, st.acc[h][2].y, st.acc[h][3].x, st.acc[h][3].y);
    dst[2 * ch1] = make_float4(st.acc[h][4].x, st.acc[h][4].y, st.acc[h][5].x, st.acc[h][5].y);
    dst[2 * ch1 + 1] = make_float4(st.acc[h][6].x, st.acc[h][6].y, st.acc[h][7].x, st.acc[h][7].y);
    if (sub == 0) {
      mine[HG * D + h] = st.m[h];
      mine[HG * D + HG + h] = st.l[h];
    }
  }
}

// Combine the NW warps' stored states (warp w at parts + w * stride floats)
// and write either bf16 rows out_rows[h * D + d], or an fp32 partial
// o_part[h * o_hstride + d] with its log2-sum-exp lse_part[h * lse_hstride].
// The caller synchronises the CTA before and after.
template <int D, int HG, int NW>
__device__ __forceinline__ void cta_combine(const float* parts, int stride, __nv_bfloat16* out_rows,
                                            float* o_part, size_t o_hstride, float* lse_part,
                                            size_t lse_hstride) {
  for (int idx = threadIdx.x; idx < HG * D; idx += NW * 32) {
    const int h = idx / D, d = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, parts[w * stride + HG * D + h]);
    float Ls = 0.f, A = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float* part = parts + w * stride;
      const float mw = part[HG * D + h];
      if (mw == -INFINITY) continue;  // this warp saw no valid row
      const float wt = ex2(mw - M);
      Ls = fmaf(part[HG * D + HG + h], wt, Ls);
      A = fmaf(part[h * D + d], wt, A);
    }
    if (out_rows != nullptr) {
      out_rows[idx] = __float2bfloat16_rn(Ls > 0.f ? A / Ls : 0.f);
    } else {
      o_part[h * o_hstride + d] = Ls > 0.f ? A / Ls : 0.f;
      if (d == 0) lse_part[h * lse_hstride] = Ls > 0.f ? M + log2f(Ls) : -INFINITY;
    }
  }
}

// Wait for the last issued use of every stage of a warp ring (only needed
// when a wait ran out and pages were left unconsumed).
template <int SW>
__device__ __forceinline__ void drain_ring(uint32_t wbar, int issued) {
  for (int s = 0; s < SW && s < issued; ++s) {
    const int last = s + ((issued - 1 - s) / SW) * SW;
    mbar_wait(wbar + 8 * s, (last / SW) & 1);
  }
}

// ============================================================================
// One CTA per (split, head group, sequence).
// PROD: warps NW..2NW-1 are producers; producer warp NW + w issues the copies
// of consumer warp w's unit stream into w's ring, so the consumers never stop
// computing to issue copies.
// ============================================================================
template <int D, int HG, int NW, int SW, int PPS, bool WIN = false, bool PROD = false>
__global__ void __launch_bounds__(NW * 32 * (PROD ? 2 : 1), PROD ? 2 : 1)
    decode_attn_kernel(const __grid_constant__ DecodeParams p) {
  using S = DecodeShape<D, HG, NW, SW, PPS, PROD>;
  extern __shared__ __align__(128) unsigned char smem[];

  const int split = blockIdx.x, hsub = blockIdx.y, b = blockIdx.z;
  const int kvh = hsub / p.nsub;
  const int head0 = kvh * p.G + (hsub % p.nsub) * HG;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool producer = PROD && warp >= NW;
  const int cw = warp % NW;  // the consumer warp whose unit stream this warp reads or fills

  int L = __ldg(p.context_lens + b);
  // The sequence's pages from the first one its sliding window reaches (WIN;
  // otherwise page 0, known before the length arrives); splits cut that range.
  const int wp0 = WIN ? window_first_key(L < 0 ? 0 : min(L, p.cap_tokens), p.window) / kPageRows : 0;
  const int pg0 = wp0 + split * p.pages_per_split;
  // The CTA's pages are cut into units of PPS consecutive pages, one unit per
  // ring stage; unit j of consumer warp cw is unit u = cw + j * NW, pages
  // pg0 + u * PPS + i.  Lane l of a chunk holds the block-table entries of
  // unit j = 32 * chunk + l.  The first two chunks are loaded together with
  // the context length (bounded by the table row and the split, not by the
  // length), so the CTA waits for one load latency before its first copy
  // instead of two.  Entries are validated where they are used.
  const int32_t* btrow = p.block_tables + (size_t)b * p.MB;
  struct Entries {
    int blk[PPS];
  };
  const bool issuer = PROD ? producer : true;  // this warp issues copies
  auto load_raw = [&](int c) {
    Entries e;
#pragma unroll
    for (int i = 0; i < PPS; ++i) {
      const int w = (cw + (c * 32 + lane) * NW) * PPS + i;  // page index within the split
      e.blk[i] = (issuer && w < p.pages_per_split && pg0 + w < p.MB) ? __ldg(btrow + pg0 + w) : 0;
    }
    return e;
  };
  const Entries raw0 = load_raw(0);
  Entries bt_nxt = load_raw(1);
  if (L < 0 || L > p.cap_tokens) {
    if (threadIdx.x == 0) set_error(PKV_ERR_BOUNDS);
    L = L < 0 ? 0 : p.cap_tokens;
  }
  const int npages = (L + kPageRows - 1) / kPageRows;
  const int n = min(npages - pg0, p.pages_per_split);  // pages of this CTA
  if (n <= 0) {
    // A split past the end of a shorter sequence leaves at once (a ragged
    // batch launches many); with one split only an empty context reaches
    // here, and its output is zero.  (In split mode the merge counts the
    // non-empty splits itself.)
    if (p.num_splits == 1)
      for (int i = threadIdx.x; i < HG * D; i += blockDim.x)
        p.out[((size_t)b * p.Hq + head0 + i / D) * D + i % D] = __float2bfloat16_rn(0.f);
    return;
  }
  // A wait that ran out earlier leaves a sticky error: do no more work until
  // the host has read and cleared it.  One thread reads the word so the whole
  // CTA takes the same branch.
  __shared__ int s_stop;
  if (threadIdx.x == 0) s_stop = *reinterpret_cast<volatile int*>(&g_error_word) == PKV_ERR_TIMEOUT;
  __syncthreads();
  if (s_stop) return;

  // ------------------------------------------------ this warp's unit stream --
  const int nu = (n + PPS - 1) / PPS;                        // units of this CTA
  const int my_n = cw < nu ? (nu - cw + NW - 1) / NW : 0;   // units cw, cw+NW, ...
  const uint32_t wring = smem_addr(smem) + cw * S::WARP_RING;
  const uint32_t wbar = smem_addr(smem) + S::BAR_OFFSET + cw * SW * 8;    // stage full
  const uint32_t ebar = smem_addr(smem) + S::EMPTY_OFFSET + cw * SW * 8;  // stage read (PROD)
  unsigned char* wring_ptr = smem + cw * S::WARP_RING;
  if (!producer && lane == 0) {
    for (int s = 0; s < SW; ++s) {
      mbar_init(wbar + 8 * s, 1);
      if (PROD) mbar_init(ebar + 8 * s, 1);
    }
    fence_barrier_init();
  }
  if (PROD)
    __syncthreads();  // the producer uses the barriers its consumer initialised
  else
    __syncwarp();

  auto validate = [&](Entries e, int c) {  // entries of pages this warp reads must lie in the pool
    const int j = c * 32 + lane;
#pragma unroll
    for (int i = 0; i < PPS; ++i)
      if (j < my_n && (cw + j * NW) * PPS + i < n && (e.blk[i] < 0 || e.blk[i] >= p.NB)) {
        set_error(PKV_ERR_BOUNDS);
        e.blk[i] = 0;  // keep every copy inside the pool
      }
    return e;
  };
  Entries bt_cur = validate(raw0, 0);
  int chunk = 0;
  const uint64_t pol = policy_evict_first();  // every page is read once
  int issued = 0;
  auto issue_next = [&]() {  // warp-uniform; units are issued in order
    const int k = issued;
    if ((k >> 5) != chunk) {
      chunk = k >> 5;
      bt_cur = validate(bt_nxt, chunk);
      bt_nxt = load_raw(chunk + 1);
    }
    const int np = min(PPS, n - (cw + k * NW) * PPS);  // pages of this unit (>= 1)
    int blk[PPS];
#pragma unroll
    for (int i = 0; i < PPS; ++i) blk[i] = __shfl_sync(0xffffffffu, bt_cur.blk[i], k & 31);
    const int s = k % SW;
    const uint32_t stage = wring + s * S::STAGE_BYTES;
    if (PROD) {
      // A thread issues bulk copies at a fixed rate whatever their size, so
      // the producer spreads a stage's 2 np copies over as many lanes: lane i
      // copies K page i, lane np + i V page i.  The byte count is posted first.
      if (lane == 0) mbar_arrive_expect_tx(wbar + 8 * s, np * 2 * S::PAGE_BYTES);
      __syncwarp();
      if (lane < 2 * np) {
        const int i = lane < np ? lane : lane - np;
        int bi = blk[0];
#pragma unroll
        for (int t = 1; t < PPS; ++t)
          if (i == t) bi = blk[t];
        const size_t off = ((size_t)bi * p.Hkv + kvh) * S::PAGE_BYTES;
        const bool is_k = lane < np;
        bulk_g2s_hint(stage + (is_k ? i : PPS + i) * S::PAGE_BYTES, (is_k ? p.k_cache : p.v_cache) + off,
                      S::PAGE_BYTES, wbar + 8 * s, pol);
      }
    } else if (lane == 0) {
      mbar_arrive_expect_tx(wbar + 8 * s, np * 2 * S::PAGE_BYTES);
#pragma unroll
      for (int i = 0; i < PPS; ++i) {
        if (i >= np) break;
        const size_t off = ((size_t)blk[i] * p.Hkv + kvh) * S::PAGE_BYTES;
        bulk_g2s_hint(stage + i * S::PAGE_BYTES, p.k_cache + off, S::PAGE_BYTES, wbar + 8 * s, pol);
        bulk_g2s_hint(stage + (PPS + i) * S::PAGE_BYTES, p.v_cache + off, S::PAGE_BYTES, wbar + 8 * s, pol);
      }
    }
    ++issued;
  };

  if (producer) {
    // ------------------------------------------------------------ producer --
    // Fill the consumer's ring in unit order; a stage is refilled once the
    // consumer has read it.  Then wait for the last copy into every stage.
    // (setmaxnreg takes one count per warpgroup: the producers are warpgroup
    // 1, the consumers warpgroup 0.)
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(S::REGS_PROD));
    for (int k = 0; k < my_n; ++k) {
      if (k >= SW && !__all_sync(0xffffffffu, mbar_wait(ebar + 8 * (k % SW), ((k / SW) - 1) & 1))) break;
      issue_next();
    }
    if (lane == 0) drain_ring<SW>(wbar, issued);
    __syncwarp();
    launch_dependents();
  } else {
    if (PROD)
      asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(S::REGS_CONS));
    else
      for (int k = 0; k < SW && k < my_n; ++k) issue_next();

    // -------------------------------------------------------- registers --
    const int rg = lane / S::LPR, sub = lane % S::LPR;
    // bf16: the lane's two 16-byte vectors of a row (D=64 odd row groups in
    // swapped order)
    const int swap = D == 64 ? (rg & 1) : 0;
    const int ch0 = sub + S::LPR * swap;        // 16-byte vector held in slot 0
    const int ch1 = sub + S::LPR * (swap ^ 1);  // and in slot 1
    float2 q2[HG][8];
    load_q<D, HG>(q2, p.q + ((size_t)b * p.Hq + head0) * D, ch0, ch1, p.scale_log2);
    LaneState<HG> st;
    st.reset();

    // valid rows counted from this CTA's first page: the sequence's, and no
    // further than the CTA's own pages
    const int rows_cta = min(L - pg0 * kPageRows, n * kPageRows);
    // rows before the window, counted the same way (<= 0 past the first split)
    const int lo_cta = WIN ? window_first_key(L, p.window) - pg0 * kPageRows : 0;
    int done = 0;
    for (int j = 0; j < my_n; ++j, ++done) {
      const int s = j % SW;
      // every lane waits (each needs the acquire); a timeout on any lane stops
      // the whole warp, which still drains its copies and joins the merge
      const bool ok = mbar_wait(wbar + 8 * s, (j / SW) & 1);
      if (!__all_sync(0xffffffffu, ok)) break;
      const unsigned char* kp = wring_ptr + s * S::STAGE_BYTES;
      attend_rows<D, HG, S::ROWS>(st, q2, kp, kp + PPS * S::PAGE_BYTES, lo_cta - (cw + j * NW) * S::ROWS,
                                  rows_cta - (cw + j * NW) * S::ROWS, rg, ch0, ch1);
      if (PROD) {
        if (j + SW < my_n) {
          // hand the stage back to the producer: order the generic-proxy reads
          // of all lanes before the copy engine's writes
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(ebar + 8 * s);
        }
      } else if (issued < my_n) {
        // the stage just read is refilled: order the generic-proxy reads of all
        // lanes before the copy engine's writes
        fence_proxy_async_smem();
        __syncwarp();
        issue_next();
      }
    }
    // Never reuse or leave the ring while one of this warp's copies may still
    // land in it (only possible after a timeout).
    if (!PROD && done < issued && lane == 0) drain_ring<SW>(wbar, issued);
    __syncwarp();
    launch_dependents();  // a merge launched after this kernel may be scheduled now

    warp_merge<D, HG>(st);
    if (PROD && done < my_n) {
      // a wait ran out: the producer may still be draining copies into this
      // ring, so the merge data go nowhere (the error word reports the call)
    } else {
      // after its last page a warp reuses its own ring for its merge data
      warp_store<D, HG>(reinterpret_cast<float*>(wring_ptr), st, rg, sub, ch0, ch1);
    }
  }
  __syncthreads();
  if (producer) return;
  const size_t row = (size_t)b * p.Hq + head0;
  const float* parts = reinterpret_cast<const float*>(smem);
  if (p.num_splits == 1)
    cta_combine<D, HG, NW>(parts, S::WARP_RING / 4, p.out + row * D, nullptr, 0, nullptr, 0);
  else  // head h of this split: o_part[((row + h) * C + split) * D + d], lse_part[(row + h) * C + split]
    cta_combine<D, HG, NW>(parts, S::WARP_RING / 4, nullptr, p.o_part + (row * p.num_splits + split) * D,
                           (size_t)p.num_splits * D, p.lse_part + row * p.num_splits + split,
                           (size_t)p.num_splits);
}

}  // namespace pkv
