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
//   * Warp NW is the producer: one lane issues 1-D bulk copies (cp.async.bulk)
//     of whole pages -- a (block, kv head) page is one contiguous 4 KB (D=128)
//     or 2 KB (D=64) run -- into a STAGES-deep shared-memory ring, completion
//     tracked by mbarriers.  Block-table entries are fetched 32 at a time.
//   * Warps 0..NW-1 consume pages round-robin.  A key row is split over
//     LPR = D/16 lanes (16 elements, two 16-byte vectors each), so a warp
//     covers 32/LPR rows per instruction and a dot product needs only
//     log2(LPR) shuffle steps.  Each lane keeps its own running max, sum and
//     fp32 accumulator for the rows it sees; warps and lanes merge once at the
//     end by log-sum-exp.
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

template <int D, int HG, int NW, int STAGES>
struct DecodeShape {
  static_assert(D == 64 || D == 128, "head_dim");
  static constexpr int LPR = D / 16;              // lanes sharing one key row
  static constexpr int RPW = 32 / LPR;            // rows per warp step
  static constexpr int TPL = kPageRows / RPW;     // rows per lane per page
  static constexpr int PAGE_BYTES = kPageRows * D * 2;
  static constexpr int STAGE_BYTES = 2 * PAGE_BYTES;  // K page + V page
  static constexpr int THREADS = (NW + 1) * 32;
  static constexpr int RING_BYTES = STAGES * STAGE_BYTES;
  static constexpr int MERGE_FLOATS = NW * HG * D + 2 * NW * HG;
  static constexpr int BAR_OFFSET = RING_BYTES + MERGE_FLOATS * 4;
  static constexpr int SMEM_BYTES = BAR_OFFSET + 2 * STAGES * 8;
};

template <int D, int HG, int NW, int STAGES>
__global__ void __launch_bounds__((NW + 1) * 32)
    decode_attn_kernel(const __grid_constant__ DecodeParams p) {
  using S = DecodeShape<D, HG, NW, STAGES>;
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

  const uint32_t ring = smem_addr(smem);
  const uint32_t bars = ring + S::BAR_OFFSET;
  auto full = [&](int s) { return bars + 8u * s; };
  auto empty = [&](int s) { return bars + 8u * (STAGES + s); };
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == NW) {
    // ------------------------------------------------------------ producer --
    const int32_t* bt = p.block_tables + (size_t)b * p.MB + pg0;
    const uint64_t pol = policy_evict_first();  // every page is read once
    int issued = 0;
    bool ok = true;
    for (int i0 = 0; i0 < n && ok; i0 += 32) {
      int blk = 0;
      if (i0 + lane < n) {
        blk = __ldg(bt + i0 + lane);
        if (blk < 0 || blk >= p.NB) {
          set_error(PKV_ERR_BOUNDS);
          blk = 0;  // keep every copy inside the pool
        }
      }
      const int cnt = min(32, n - i0);
      for (int j = 0; j < cnt; ++j) {
        const int bj = __shfl_sync(0xffffffffu, blk, j);
        const int i = i0 + j, s = i % STAGES;
        if (lane == 0) {
          if (i >= STAGES) ok = mbar_wait(empty(s), ((i / STAGES) & 1) ^ 1);
          if (ok) {
            const size_t off = ((size_t)bj * p.Hkv + kvh) * S::PAGE_BYTES;
            mbar_arrive_expect_tx(full(s), S::STAGE_BYTES);
            bulk_g2s_hint(ring + s * S::STAGE_BYTES, p.k_cache + off, S::PAGE_BYTES, full(s), pol);
            bulk_g2s_hint(ring + s * S::STAGE_BYTES + S::PAGE_BYTES, p.v_cache + off,
                          S::PAGE_BYTES, full(s), pol);
            ++issued;
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
      }
    }
    // Do not leave while a copy into this CTA's shared memory may be in
    // flight: wait for the last issued use of every stage to land.
    if (lane == 0) {
      for (int s = 0; s < STAGES && s < issued; ++s) {
        const int last = s + ((issued - 1 - s) / STAGES) * STAGES;
        mbar_wait(full(s), (last / STAGES) & 1);
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers --
  const int rg = lane / S::LPR, sub = lane % S::LPR;
  const int swap = (D == 64) ? (rg & 1) : 0;
  const int ch0 = sub + S::LPR * swap;        // 16-byte vector held in slot 0
  const int ch1 = sub + S::LPR * (swap ^ 1);  // and in slot 1

  float qf[HG][16];
#pragma unroll
  for (int h = 0; h < HG; ++h) {
    const uint4* qrow = reinterpret_cast<const uint4*>(p.q + ((size_t)b * p.Hq + head0 + h) * D);
    widen8(__ldg(qrow + ch0), qf[h]);
    widen8(__ldg(qrow + ch1), qf[h] + 8);
#pragma unroll
    for (int e = 0; e < 16; ++e) qf[h][e] *= p.scale_log2;
  }

  float m[HG], l[HG], acc[HG][16];
#pragma unroll
  for (int h = 0; h < HG; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
#pragma unroll
    for (int e = 0; e < 16; ++e) acc[h][e] = 0.f;
  }

  const int L_local = L - pg0 * kPageRows;  // valid rows counted from this CTA's first page
  for (int i = warp; i < n; i += NW) {
    const int s = i % STAGES;
    // every lane waits (each needs the acquire); a timeout on any lane stops
    // the whole warp, which still joins the merge below
    const bool ok = mbar_wait(full(s), (i / STAGES) & 1);
    if (!__all_sync(0xffffffffu, ok)) break;
    const unsigned char* kp = smem + s * S::STAGE_BYTES;
    const unsigned char* vp = kp + S::PAGE_BYTES;
    const int row0 = i * kPageRows;

    float sc[S::TPL][HG];
#pragma unroll
    for (int t = 0; t < S::TPL; ++t) {
      const int r = rg + t * S::RPW;
      const uint4* krow = reinterpret_cast<const uint4*>(kp + r * D * 2);
      float kf[16];
      widen8(krow[ch0], kf);
      widen8(krow[ch1], kf + 8);
#pragma unroll
      for (int h = 0; h < HG; ++h) {
        float d0 = 0.f, d1 = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          d0 = fmaf(qf[h][e], kf[e], d0);
          d1 = fmaf(qf[h][8 + e], kf[8 + e], d1);
        }
        sc[t][h] = d0 + d1;
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
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[h][e] *= alpha;
      }
    }
#pragma unroll
    for (int t = 0; t < S::TPL; ++t) {
      if (!valid[t]) continue;  // canary / stale rows are never touched
      const int r = rg + t * S::RPW;
      const uint4* vrow = reinterpret_cast<const uint4*>(vp + r * D * 2);
      float vf[16];
      widen8(vrow[ch0], vf);
      widen8(vrow[ch1], vf + 8);
#pragma unroll
      for (int h = 0; h < HG; ++h) {
        const float pr = ex2(sc[t][h] - m[h]);
        l[h] += pr;
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[h][e] = fmaf(pr, vf[e], acc[h][e]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty(s));
  }

  // ---- merge the row groups of this warp (lanes with the same D-slice) ----
#pragma unroll
  for (int off = S::LPR; off < 32; off <<= 1) {
    const int flip = (D == 64 && off == S::LPR) ? 8 : 0;  // partner keeps the other order
#pragma unroll
    for (int h = 0; h < HG; ++h) {
      const float mo = __shfl_xor_sync(0xffffffffu, m[h], off);
      const float lo = __shfl_xor_sync(0xffffffffu, l[h], off);
      const float mn = fmaxf(m[h], mo);
      const float a = (mn == -INFINITY) ? 0.f : ex2(m[h] - mn);
      const float c = (mn == -INFINITY) ? 0.f : ex2(mo - mn);
      float recv[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) recv[e] = __shfl_xor_sync(0xffffffffu, acc[h][e ^ flip], off);
#pragma unroll
      for (int e = 0; e < 16; ++e) acc[h][e] = acc[h][e] * a + recv[e] * c;
      l[h] = l[h] * a + lo * c;
      m[h] = mn;
    }
  }

  // ---- merge the warps through shared memory -------------------------------
  float* sm_acc = reinterpret_cast<float*>(smem + S::RING_BYTES);  // [NW][HG][D]
  float* sm_m = sm_acc + NW * HG * D;                               // [NW][HG]
  float* sm_l = sm_m + NW * HG;
  if (rg == 0) {  // lanes 0..LPR-1 hold the warp's result in natural order
#pragma unroll
    for (int h = 0; h < HG; ++h) {
      float4* dst = reinterpret_cast<float4*>(sm_acc + (warp * HG + h) * D);
      dst[2 * ch0] = make_float4(acc[h][0], acc[h][1], acc[h][2], acc[h][3]);
      dst[2 * ch0 + 1] = make_float4(acc[h][4], acc[h][5], acc[h][6], acc[h][7]);
      dst[2 * ch1] = make_float4(acc[h][8], acc[h][9], acc[h][10], acc[h][11]);
      dst[2 * ch1 + 1] = make_float4(acc[h][12], acc[h][13], acc[h][14], acc[h][15]);
      if (sub == 0) {
        sm_m[warp * HG + h] = m[h];
        sm_l[warp * HG + h] = l[h];
      }
    }
  }
  named_barrier_sync(1, NW * 32);
  for (int idx = threadIdx.x; idx < HG * D; idx += NW * 32) {
    const int h = idx / D, d = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, sm_m[w * HG + h]);
    float Ls = 0.f, A = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float mw = sm_m[w * HG + h];
      if (mw == -INFINITY) continue;  // this warp saw no valid row
      const float wt = ex2(mw - M);
      Ls = fmaf(sm_l[w * HG + h], wt, Ls);
      A = fmaf(sm_acc[(w * HG + h) * D + d], wt, A);
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
