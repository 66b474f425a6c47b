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
//   * One CTA = (sequence b, a group of HG query heads sharing one kv head,
//     a range of pages).  The HG query rows live in registers, so every K/V
//     byte is read from HBM once per group (grouped-query reuse).
//   * Every warp feeds itself: lane 0 issues 1-D bulk copies (cp.async.bulk)
//     of whole pages -- a (block, kv head) page is one contiguous 4 KB (D=128)
//     or 2 KB (D=64) run -- into the warp's own SW-stage shared-memory ring,
//     completion tracked by one mbarrier per stage.  A warp refills a stage
//     as soon as it has read it, so no cross-warp hand-off is needed and no
//     warp is spent on copies.  Block-table entries are fetched 32 at a time,
//     one chunk ahead.
//   * Two CTAs per SM (shared-memory carveout at its maximum) keep
//     2 x NW x SW pages -- about 192 KB -- in flight per SM, which is what
//     Little's law asks for at full HBM bandwidth.
//   * A key row is split over LPR = D/16 lanes (16 elements, two 16-byte
//     vectors each), so a warp covers 32/LPR rows per instruction and a dot
//     product needs only log2(LPR) shuffle steps.  Products and P.V updates
//     use packed fp32 (FFMA2) on element pairs.  Each lane keeps its own
//     running max, sum and fp32 accumulator; lanes and warps merge once at
//     the end by log-sum-exp.
//   * Split mode (num_splits > 1): each CTA writes its normalised partial and
//     its log2-domain log-sum-exp; lse_merge_kernel combines them.
//   * Shared-memory reads are conflict-free: for D=128 the 8 lanes of a row
//     read 128 contiguous bytes per phase; for D=64 odd row groups read their
//     two vectors in swapped order, and their q / accumulator registers are
//     kept in that swapped order too.
#pragma once
#include "pkv_common.cuh"

namespace pkv {

constexpr int kPageRows = 16;  // block_size supported by the attention kernels

struct DecodeParams {
  __nv_bfloat16* out;            // [B][Hq][D]
  float* o_part;                 // [B][Hq][C][D]   split mode
  float* lse_part;               // [B][Hq][C]      split mode, log2 domain
  const __nv_bfloat16* q;        // [B][Hq][D]
  const unsigned char* k_cache;  // [NB][Hkv][16][D] bf16
  const unsigned char* v_cache;
  const int32_t* block_tables;   // [B][MB]
  const int32_t* context_lens;   // [B]
  int32_t B, Hq, Hkv, NB, MB;
  int32_t G;                     // Hq / Hkv
  int32_t nsub;                  // G / HG head groups per kv head
  int32_t pages_per_split;
  int32_t num_splits;            // 1: write bf16 output directly
  int32_t cap_tokens;            // longest context this launch can hold
  float scale_log2;              // scale * log2(e)
};

template <int D, int HG, int NW, int SW>
struct DecodeShape {
  static_assert(D == 64 || D == 128, "head_dim");
  static constexpr int LPR = D / 16;              // lanes sharing one key row
  static constexpr int RPW = 32 / LPR;            // rows per warp step
  static constexpr int TPL = kPageRows / RPW;     // rows per lane per page
  static constexpr int PAGE_BYTES = kPageRows * D * 2;
  static constexpr int STAGE_BYTES = 2 * PAGE_BYTES;  // K page + V page
  static constexpr int THREADS = NW * 32;
  static constexpr int WARP_RING = SW * STAGE_BYTES;
  static constexpr int RING_BYTES = NW * WARP_RING;
  // after its last page a warp reuses its own ring for the merge data
  static constexpr int MERGE_BYTES = (HG * D + 2 * HG) * 4;
  static_assert(MERGE_BYTES <= WARP_RING, "merge data must fit the warp's ring");
  static constexpr int BAR_OFFSET = RING_BYTES;
  static constexpr int SMEM_BYTES = BAR_OFFSET + NW * SW * 8;
};

__device__ __forceinline__ float2 widen2(uint32_t w) {
  return make_float2(bf16lo_to_f32(w), bf16hi_to_f32(w));
}

template <int D, int HG, int NW, int SW>
__global__ void __launch_bounds__(NW * 32)
    decode_attn_kernel(const __grid_constant__ DecodeParams p) {
  using S = DecodeShape<D, HG, NW, SW>;
  extern __shared__ __align__(128) unsigned char smem[];

  const int split = blockIdx.x, hsub = blockIdx.y, b = blockIdx.z;
  const int kvh = hsub / p.nsub;
  const int head0 = kvh * p.G + (hsub % p.nsub) * HG;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  int L = __ldg(p.context_lens + b);
  if (L < 0 || L > p.cap_tokens) {
    if (threadIdx.x == 0) set_error(PKV_ERR_BOUNDS);
    L = L < 0 ? 0 : p.cap_tokens;
  }
  const int npages = (L + kPageRows - 1) / kPageRows;
  const int pg0 = split * p.pages_per_split;
  const int n = min(npages - pg0, p.pages_per_split);  // pages of this CTA
  // A wait that ran out earlier leaves a sticky error: do no more work until
  // the host has read and cleared it.  One thread reads the word so the whole
  // CTA takes the same branch.
  __shared__ int s_stop;
  if (threadIdx.x == 0) s_stop = *reinterpret_cast<volatile int*>(&g_error_word) == PKV_ERR_TIMEOUT;
  __syncthreads();
  if (s_stop) return;
  if (n <= 0) {
    // Only an empty context reaches here with one split: its output is zero.
    // (In split mode the merge counts the non-empty splits itself.)
    if (p.num_splits == 1)
      for (int i = threadIdx.x; i < HG * D; i += blockDim.x)
        p.out[((size_t)b * p.Hq + head0 + i / D) * D + i % D] = __float2bfloat16_rn(0.f);
    return;
  }

  // ------------------------------------------------ this warp's page stream --
  const int my_n = warp < n ? (n - warp + NW - 1) / NW : 0;  // pages warp, warp+NW, ...
  const uint32_t wring = smem_addr(smem) + warp * S::WARP_RING;
  const uint32_t wbar = smem_addr(smem) + S::BAR_OFFSET + warp * SW * 8;
  unsigned char* wring_ptr = smem + warp * S::WARP_RING;
  if (lane == 0) {
    for (int s = 0; s < SW; ++s) mbar_init(wbar + 8 * s, 1);
    fence_barrier_init();
  }
  __syncwarp();

  const int32_t* btw = p.block_tables + (size_t)b * p.MB + pg0 + warp;  // entry of page j: btw[j*NW]
  auto load_chunk = [&](int c) {
    const int j = c * 32 + lane;
    int blk = 0;
    if (j < my_n) {
      blk = __ldg(btw + (size_t)j * NW);
      if (blk < 0 || blk >= p.NB) {
        set_error(PKV_ERR_BOUNDS);
        blk = 0;  // keep every copy inside the pool
      }
    }
    return blk;
  };
  int bt_cur = load_chunk(0), bt_nxt = load_chunk(1), chunk = 0;
  const uint64_t pol = policy_evict_first();  // every page is read once
  int issued = 0;
  auto issue_next = [&]() {  // warp-uniform; pages are issued in order
    const int k = issued;
    if ((k >> 5) != chunk) {
      bt_cur = bt_nxt;
      chunk = k >> 5;
      bt_nxt = load_chunk(chunk + 1);
    }
    const int blk = __shfl_sync(0xffffffffu, bt_cur, k & 31);
    if (lane == 0) {
      const int s = k % SW;
      const size_t off = ((size_t)blk * p.Hkv + kvh) * S::PAGE_BYTES;
      mbar_arrive_expect_tx(wbar + 8 * s, S::STAGE_BYTES);
      bulk_g2s_hint(wring + s * S::STAGE_BYTES, p.k_cache + off, S::PAGE_BYTES, wbar + 8 * s, pol);
      bulk_g2s_hint(wring + s * S::STAGE_BYTES + S::PAGE_BYTES, p.v_cache + off, S::PAGE_BYTES,
                    wbar + 8 * s, pol);
    }
    ++issued;
  };
  for (int k = 0; k < SW && k < my_n; ++k) issue_next();

  // ---------------------------------------------------------- registers --
  const int rg = lane / S::LPR, sub = lane % S::LPR;
  const int swap = (D == 64) ? (rg & 1) : 0;
  const int ch0 = sub + S::LPR * swap;        // 16-byte vector held in slot 0
  const int ch1 = sub + S::LPR * (swap ^ 1);  // and in slot 1

  float2 q2[HG][8];  // the lane's 16 q elements as 8 pairs, pre-scaled
#pragma unroll
  for (int h = 0; h < HG; ++h) {
    const uint4* qrow = reinterpret_cast<const uint4*>(p.q + ((size_t)b * p.Hq + head0 + h) * D);
    const uint4 a = __ldg(qrow + ch0), c = __ldg(qrow + ch1);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
    const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
#pragma unroll
    for (int e = 0; e < 8; ++e) q2[h][e] = __fmul2_rn(widen2(w[e]), sc2);
  }

  float m[HG], l[HG];
  float2 acc2[HG][8];
#pragma unroll
  for (int h = 0; h < HG; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc2[h][e] = make_float2(0.f, 0.f);
  }

  const int L_local = L - pg0 * kPageRows;  // valid rows counted from this CTA's first page
  int done = 0;
  for (int j = 0; j < my_n; ++j, ++done) {
    const int s = j % SW;
    // every lane waits (each needs the acquire); a timeout on any lane stops
    // the whole warp, which still drains its copies and joins the merge
    const bool ok = mbar_wait(wbar + 8 * s, (j / SW) & 1);
    if (!__all_sync(0xffffffffu, ok)) break;
    const unsigned char* kp = wring_ptr + s * S::STAGE_BYTES;
    const unsigned char* vp = kp + S::PAGE_BYTES;
    const int row0 = (warp + j * NW) * kPageRows;

    float sc[S::TPL][HG];
#pragma unroll
    for (int t = 0; t < S::TPL; ++t) {
      const int r = rg + t * S::RPW;
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
    for (int off = S::LPR / 2; off >= 1; off >>= 1)
#pragma unroll
      for (int t = 0; t < S::TPL; ++t)
#pragma unroll
        for (int h = 0; h < HG; ++h) sc[t][h] += __shfl_xor_sync(0xffffffffu, sc[t][h], off);

    bool valid[S::TPL];
#pragma unroll
    for (int t = 0; t < S::TPL; ++t) valid[t] = row0 + rg + t * S::RPW < L_local;

    float mp[HG];
    bool grow = false;
#pragma unroll
    for (int h = 0; h < HG; ++h) {
      mp[h] = -INFINITY;
#pragma unroll
      for (int t = 0; t < S::TPL; ++t)
        if (valid[t]) mp[h] = fmaxf(mp[h], sc[t][h]);
      grow |= mp[h] > m[h];
    }
    if (__any_sync(0xffffffffu, grow)) {
#pragma unroll
      for (int h = 0; h < HG; ++h) {
        const float mn = fmaxf(m[h], mp[h]);
        const float alpha = (mn == -INFINITY) ? 1.f : ex2(m[h] - mn);
        m[h] = mn;
        l[h] *= alpha;
        const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc2[h][e] = __fmul2_rn(acc2[h][e], a2);
      }
    }
#pragma unroll
    for (int t = 0; t < S::TPL; ++t) {
      if (!valid[t]) continue;  // canary / stale rows are never touched
      const int r = rg + t * S::RPW;
      const uint4* vrow = reinterpret_cast<const uint4*>(vp + r * D * 2);
      const uint4 va = vrow[ch0], vb = vrow[ch1];
      const float2 v2[8] = {widen2(va.x), widen2(va.y), widen2(va.z), widen2(va.w),
                            widen2(vb.x), widen2(vb.y), widen2(vb.z), widen2(vb.w)};
#pragma unroll
      for (int h = 0; h < HG; ++h) {
        const float pr = ex2(sc[t][h] - m[h]);
        l[h] += pr;
        const float2 pp = make_float2(pr, pr);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc2[h][e] = __ffma2_rn(pp, v2[e], acc2[h][e]);
      }
    }
    if (issued < my_n) {
      // the stage just read is refilled: order the generic-proxy reads of all
      // lanes before the copy engine's writes
      fence_proxy_async_smem();
      __syncwarp();
      issue_next();
    }
  }
  // Never reuse or leave the ring while one of this warp's copies may still
  // land in it (only possible after a timeout): wait for the last issued use
  // of every stage.
  if (done < issued && lane == 0) {
    for (int s = 0; s < SW && s < issued; ++s) {
      const int last = s + ((issued - 1 - s) / SW) * SW;
      mbar_wait(wbar + 8 * s, (last / SW) & 1);
    }
  }
  __syncwarp();

  // ---- merge the row groups of this warp (lanes with the same D-slice) ----
#pragma unroll
  for (int off = S::LPR; off < 32; off <<= 1) {
    const int flip = (D == 64 && off == S::LPR) ? 4 : 0;  // partner keeps the other order
#pragma unroll
    for (int h = 0; h < HG; ++h) {
      const float mo = __shfl_xor_sync(0xffffffffu, m[h], off);
      const float lo = __shfl_xor_sync(0xffffffffu, l[h], off);
      const float mn = fmaxf(m[h], mo);
      const float a = (mn == -INFINITY) ? 0.f : ex2(m[h] - mn);
      const float c = (mn == -INFINITY) ? 0.f : ex2(mo - mn);
      float2 recv[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        recv[e].x = __shfl_xor_sync(0xffffffffu, acc2[h][e ^ flip].x, off);
        recv[e].y = __shfl_xor_sync(0xffffffffu, acc2[h][e ^ flip].y, off);
      }
      const float2 a2 = make_float2(a, a), c2 = make_float2(c, c);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc2[h][e] = __ffma2_rn(acc2[h][e], a2, __fmul2_rn(recv[e], c2));
      l[h] = l[h] * a + lo * c;
      m[h] = mn;
    }
  }

  // ---- merge the warps through shared memory (each warp's own ring) -------
  {
    float* mine = reinterpret_cast<float*>(wring_ptr);  // [HG][D] acc, [HG] m, [HG] l
    if (rg == 0) {  // lanes 0..LPR-1 hold the warp's result in natural order
#pragma unroll
      for (int h = 0; h < HG; ++h) {
        float4* dst = reinterpret_cast<float4*>(mine + h * D);
        dst[2 * ch0] = make_float4(acc2[h][0].x, acc2[h][0].y, acc2[h][1].x, acc2[h][1].y);
        dst[2 * ch0 + 1] = make_float4(acc2[h][2].x, acc2[h][2].y, acc2[h][3].x, acc2[h][3].y);
        dst[2 * ch1] = make_float4(acc2[h][4].x, acc2[h][4].y, acc2[h][5].x, acc2[h][5].y);
        dst[2 * ch1 + 1] = make_float4(acc2[h][6].x, acc2[h][6].y, acc2[h][7].x, acc2[h][7].y);
        if (sub == 0) {
          mine[HG * D + h] = m[h];
          mine[HG * D + HG + h] = l[h];
        }
      }
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < HG * D; idx += NW * 32) {
    const int h = idx / D, d = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w)
      M = fmaxf(M, reinterpret_cast<const float*>(smem + w * S::WARP_RING)[HG * D + h]);
    float Ls = 0.f, A = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float* part = reinterpret_cast<const float*>(smem + w * S::WARP_RING);
      const float mw = part[HG * D + h];
      if (mw == -INFINITY) continue;  // this warp saw no valid row
      const float wt = ex2(mw - M);
      Ls = fmaf(part[HG * D + HG + h], wt, Ls);
      A = fmaf(part[h * D + d], wt, A);
    }
    const size_t row = (size_t)b * p.Hq + head0 + h;
    if (p.num_splits == 1) {
      p.out[row * D + d] = __float2bfloat16_rn(Ls > 0.f ? A / Ls : 0.f);
    } else {
      const size_t prow = row * p.num_splits + split;
      p.o_part[prow * D + d] = Ls > 0.f ? A / Ls : 0.f;
      if (d == 0) p.lse_part[prow] = Ls > 0.f ? M + log2f(Ls) : -INFINITY;
    }
  }
}

// ----------------------------------------------------------------------------
// Log-sum-exp merge of split partials (log2 domain):
//   out = sum_c 2^{lse_c - M} o_c / sum_c 2^{lse_c - M},  M = max_c lse_c,
// over the splits that hold at least one key of the sequence.
// ----------------------------------------------------------------------------
struct MergeParams {
  __nv_bfloat16* out;         // [B][Hq][D]
  const float* o_part;        // [B][Hq][C][D]
  const float* lse_part;      // [B][Hq][C]
  const int32_t* context_lens;
  int32_t Hq, num_splits, pages_per_split, cap_tokens;
};

template <int D>
__global__ void __launch_bounds__(D) lse_merge_kernel(const __grid_constant__ MergeParams p) {
  const int h = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  int L = __ldg(p.context_lens + b);
  L = L < 0 ? 0 : (L > p.cap_tokens ? p.cap_tokens : L);
  const int npages = (L + kPageRows - 1) / kPageRows;
  const int nval = (npages + p.pages_per_split - 1) / p.pages_per_split;
  const size_t row = (size_t)b * p.Hq + h;
  const float* lse = p.lse_part + row * p.num_splits;
  const float* o = p.o_part + row * p.num_splits * D;
  float M = -INFINITY;
  for (int c = 0; c < nval; ++c) M = fmaxf(M, lse[c]);
  float ws = 0.f, a = 0.f;
  for (int c = 0; c < nval; ++c) {
    if (lse[c] == -INFINITY) continue;
    const float w = ex2(lse[c] - M);
    ws += w;
    a = fmaf(w, o[(size_t)c * D + d], a);
  }
  p.out[row * D + d] = __float2bfloat16_rn(ws > 0.f ? a / ws : 0.f);
}

}  // namespace pkv
