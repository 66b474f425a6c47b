// prefill_attn.cuh -- causal chunked prefill over the paged KV cache on the
// tcgen05 tensor cores.
//
// Method: a chunk of new queries attends to the cached context plus its own
// causal prefix; S = Q.K^T, online softmax (running max / running sum) and
// O += P.V run tile by tile so the score matrix never leaves the chip
// ("从零构建CUDA推理引擎：Tiny-Infer项目的技术深度解析", sections
// "Flash Attention：内存与计算的重平衡" and "分页KV缓存：借鉴操作系统的内存管理";
// "5 Fun Projects for LLM Inference Engineering", section 2).  Unlike decode,
// this is a dense contraction (about 1300 flop per byte at 4096 context), so
// it belongs on the tensor cores.
//
// B200 design (one CTA per SM):
//   * Tile = 128 query rows x 128 keys.  The G query heads of one kv head are
//     packed into the rows (row = position * G + head), so every K/V tile
//     loaded feeds all of them.
//   * Warp 0 (one lane) loads Q once and K/V tiles through a 3-stage ring with
//     tiled TMA: each 16-key page of the paged cache is one 16 x 64-element
//     box per head-dim half, landing in the 128-byte-swizzled layout the MMA
//     reads.  A page beyond the context is addressed out of range, so TMA
//     fills it with zeros.
//   * Warp 1 (one lane) issues tcgen05.mma: S_j = Q K_j^T into one of two TMEM
//     score buffers, then O += P_{j-1} V_{j-1} with P read straight from TMEM
//     (bf16, written over the score buffer it came from) and V from shared
//     memory as an MN-major operand.  tcgen05.commit signals each stage.
//   * Warps 4-7 (one warpgroup, thread = TMEM lane = query row) load a score
//     row, apply the causal mask on the diagonal tiles only, update the
//     running max and sum, and write P back to TMEM.  O is rescaled in TMEM
//     only when the running max grows by more than 2^8 (exact after the final
//     division by the row sum).  The same warps finish with O / l to global.
//   * TMEM: two 128-column score buffers and one 128-column O accumulator.
//   * Every mbarrier wait is bounded; on a timeout each role stops, in-flight
//     copies and MMAs are waited for, and TMEM is released.
#pragma once
#include "pkv_common.cuh"
#include "tcgen05.cuh"

namespace pkv {

struct PrefillParams {
  __nv_bfloat16* out;            // [sumQ][Hq][128]
  const int32_t* query_start_loc;  // [B+1]
  const int32_t* block_tables;   // [B][MB]
  const int32_t* context_lens;   // [B]
  int32_t B, Hq, Hkv, NB, MB, G, sumQ;
  float scale_log2;              // scale * log2(e), >= 0
};

namespace pf {
constexpr int D = 128;
constexpr int BM = 128;                 // query rows per tile
constexpr int BN = 128;                 // keys per tile (8 pages)
constexpr int STAGES = 3;
constexpr int HALF_BYTES = 128 * 128;   // 128 rows x 64 bf16 (one head-dim half)
constexpr int TILE_BYTES = 2 * HALF_BYTES;
constexpr int PAGE_BOX_BYTES = 16 * 128;  // one page, one half
constexpr int Q_OFF = 0;
constexpr int K_OFF = Q_OFF + TILE_BYTES;
constexpr int V_OFF = K_OFF + STAGES * TILE_BYTES;
constexpr int BAR_OFF = V_OFF + STAGES * TILE_BYTES;
// barriers
constexpr int B_Q = 0;
constexpr int B_KFULL = 1;
constexpr int B_VFULL = B_KFULL + STAGES;
constexpr int B_KVEMPTY = B_VFULL + STAGES;
constexpr int B_SFULL = B_KVEMPTY + STAGES;  // 2
constexpr int B_PFULL = B_SFULL + 2;         // 2
constexpr int B_OREADY = B_PFULL + 2;
constexpr int B_MMADONE = B_OREADY + 1;
constexpr int NUM_BARS = B_MMADONE + 1;
constexpr int TMEM_SLOT_OFF = BAR_OFF + NUM_BARS * 8;
constexpr int SMEM_BYTES = TMEM_SLOT_OFF + 16 + 1024;  // + slack to align the base to 1 KB
constexpr int THREADS = 256;
constexpr int TMEM_COLS = 512;
constexpr int S_BUF_COLS = 128;  // score buffer i starts at column i * 128
constexpr int O_COL = 256;
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units: rescale O when the max grows by > 2^8
}  // namespace pf

__global__ void __launch_bounds__(pf::THREADS, 1)
    prefill_attn_kernel(const __grid_constant__ PrefillParams p, const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* sbase = smem_raw + (base - raw);

  const int mt = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.G, PPT = pf::BM / G;  // query positions per tile

  const int qs = __ldg(p.query_start_loc + b);
  const int Qb = __ldg(p.query_start_loc + b + 1) - qs;
  const int L = __ldg(p.context_lens + b);
  const int p0 = mt * PPT;

  __shared__ int s_flag;
  if (threadIdx.x == 0) {
    int f = *reinterpret_cast<volatile int*>(&g_error_word) == PKV_ERR_TIMEOUT;
    if (Qb < 0 || L < Qb || L > p.MB * 16 || qs < 0 || qs + Qb > p.sumQ) {
      set_error(PKV_ERR_BOUNDS);
      f = 1;
    }
    s_flag = f;
  }
  __syncthreads();
  if (s_flag || p0 >= Qb) return;

  const int last_pos = min(p0 + PPT, Qb) - 1;
  const int kv_end = L - Qb + last_pos + 1;  // keys the last valid row can see
  const int n_tiles = (kv_end + pf::BN - 1) / pf::BN;
  const int npages = (L + 15) / 16;

  auto bar = [&](int i) { return base + pf::BAR_OFF + 8u * i; };
  if (threadIdx.x == 0) {
    mbar_init(bar(pf::B_Q), 1);
    for (int s = 0; s < pf::STAGES; ++s) {
      mbar_init(bar(pf::B_KFULL + s), 1);
      mbar_init(bar(pf::B_VFULL + s), 1);
      mbar_init(bar(pf::B_KVEMPTY + s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(pf::B_SFULL + i), 1);
      mbar_init(bar(pf::B_PFULL + i), 4);  // one arrival per softmax warp
    }
    mbar_init(bar(pf::B_OREADY), 1);
    mbar_init(bar(pf::B_MMADONE), 1);
    fence_barrier_init();
  }
  if (warp == 2) {
    tc::alloc(base + pf::TMEM_SLOT_OFF, pf::TMEM_COLS);
    tc::relinquish_alloc_permit();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sbase + pf::TMEM_SLOT_OFF);

  if (warp == 0) {
    // ---------------------------------------------------------- TMA loads --
    if (lane == 0) {
      tc::prefetch_tensormap(&tm_q);
      tc::prefetch_tensormap(&tm_k);
      tc::prefetch_tensormap(&tm_v);
      mbar_arrive_expect_tx(bar(pf::B_Q), pf::TILE_BYTES);
      tc::tma_load_3d(base + pf::Q_OFF, &tm_q, 0, kvh * G, qs + p0, bar(pf::B_Q));
      tc::tma_load_3d(base + pf::Q_OFF + pf::HALF_BYTES, &tm_q, 64, kvh * G, qs + p0, bar(pf::B_Q));
    }
    const int32_t* bt = p.block_tables + (size_t)b * p.MB;
    int issued = 0;
    for (int j = 0; j < n_tiles; ++j) {
      const int s = j % pf::STAGES;
      if (j >= pf::STAGES) {
        bool ok = true;
        if (lane == 0) ok = mbar_wait(bar(pf::B_KVEMPTY + s), ((j / pf::STAGES) - 1) & 1);
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      }
      int blk = p.NB;  // out of range: TMA fills the page with zeros
      if (lane < 8) {
        const int pg = j * 8 + lane;
        if (pg < npages) {
          blk = __ldg(bt + pg);
          if (blk < 0 || blk >= p.NB) {
            set_error(PKV_ERR_BOUNDS);
            blk = p.NB;
          }
        }
      }
      if (lane == 0) {
        mbar_arrive_expect_tx(bar(pf::B_KFULL + s), pf::TILE_BYTES);
        mbar_arrive_expect_tx(bar(pf::B_VFULL + s), pf::TILE_BYTES);
      }
      __syncwarp();
      if (lane < 8) {
        const uint32_t kd = base + pf::K_OFF + s * pf::TILE_BYTES + lane * pf::PAGE_BOX_BYTES;
        const uint32_t vd = base + pf::V_OFF + s * pf::TILE_BYTES + lane * pf::PAGE_BOX_BYTES;
        tc::tma_load_4d(kd, &tm_k, 0, 0, kvh, blk, bar(pf::B_KFULL + s));
        tc::tma_load_4d(kd + pf::HALF_BYTES, &tm_k, 64, 0, kvh, blk, bar(pf::B_KFULL + s));
        tc::tma_load_4d(vd, &tm_v, 0, 0, kvh, blk, bar(pf::B_VFULL + s));
        tc::tma_load_4d(vd + pf::HALF_BYTES, &tm_v, 64, 0, kvh, blk, bar(pf::B_VFULL + s));
      }
      ++issued;
    }
    // leave no copy in flight: wait for the last issued use of every stage
    if (lane == 0) {
      mbar_wait(bar(pf::B_Q), 0);
      for (int s = 0; s < pf::STAGES && s < issued; ++s) {
        const int last = s + ((issued - 1 - s) / pf::STAGES) * pf::STAGES;
        mbar_wait(bar(pf::B_KFULL + s), (last / pf::STAGES) & 1);
        mbar_wait(bar(pf::B_VFULL + s), (last / pf::STAGES) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA ------
    constexpr uint32_t IDESC_S = tc::idesc_bf16_f32(pf::BM, pf::BN, false, false);
    constexpr uint32_t IDESC_PV = tc::idesc_bf16_f32(pf::BM, pf::D, false, true);
    const uint32_t q_s = base + pf::Q_OFF;
    bool ok = __all_sync(0xffffffffu, mbar_wait(bar(pf::B_Q), 0));
    // the page holding the sequence's last key, if it is only partly valid
    const int tail_rows = L % 16;
    const int tail_page = (L - 1) / 16;

    auto pv = [&](int t) -> bool {
      const int st = t % pf::STAGES;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(pf::B_PFULL + (t & 1)), (t >> 1) & 1))) return false;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(pf::B_VFULL + st), (t / pf::STAGES) & 1))) return false;
      tc::fence_after_sync();
      const uint32_t v_s = base + pf::V_OFF + st * pf::TILE_BYTES;
      if (tail_rows != 0 && tail_page / 8 == t) {
        // rows past the end of the context hold stale data that a zero
        // probability would not cancel if it were NaN: clear them
        unsigned char* vp = sbase + pf::V_OFF + st * pf::TILE_BYTES + (tail_page % 8) * pf::PAGE_BOX_BYTES;
        const int nvec = (16 - tail_rows) * 8;  // 16-byte vectors per half
        for (int i = lane; i < 2 * nvec; i += 32) {
          const int half = i / nvec, k = i % nvec;
          *reinterpret_cast<uint4*>(vp + half * pf::HALF_BYTES + tail_rows * 128 + k * 16) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
        __syncwarp();
      }
      if (lane == 0) {
        const uint32_t p_t = tmem + (t & 1) * pf::S_BUF_COLS;
#pragma unroll
        for (int kk = 0; kk < pf::BN / 16; ++kk) {
          const uint64_t bd = tc::smem_desc_sw128(v_s + kk * 2048, pf::HALF_BYTES, 1024);
          tc::mma_ts(tmem + pf::O_COL, p_t + kk * 8, bd, IDESC_PV, (t > 0 || kk > 0) ? 1u : 0u);
        }
        tc::commit(bar(pf::B_KVEMPTY + st));
        tc::commit(bar(pf::B_OREADY));
      }
      __syncwarp();
      return true;
    };

    for (int j = 0; j < n_tiles && ok; ++j) {
      const int st = j % pf::STAGES;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(pf::B_KFULL + st), (j / pf::STAGES) & 1))) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      if (lane == 0) {
        const uint32_t k_s = base + pf::K_OFF + st * pf::TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < pf::D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * pf::HALF_BYTES + (kk & 3) * 32;
          const uint64_t ad = tc::smem_desc_sw128(q_s + off, 16, 1024);
          const uint64_t bd = tc::smem_desc_sw128(k_s + off, 16, 1024);
          tc::mma_ss(tmem + (j & 1) * pf::S_BUF_COLS, ad, bd, IDESC_S, kk > 0 ? 1u : 0u);
        }
        tc::commit(bar(pf::B_SFULL + (j & 1)));
      }
      __syncwarp();
      if (j >= 1 && !pv(j - 1)) ok = false;
    }
    if (ok) pv(n_tiles - 1);
    // all MMAs of this CTA retired before TMEM is released
    if (lane == 0) {
      tc::commit(bar(pf::B_MMADONE));
      mbar_wait(bar(pf::B_MMADONE), 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // --------------------------------------------- softmax and epilogue -----
    const int wq = warp - 4;                     // TMEM lane quarter of this warp
    const int r = wq * 32 + lane;                // query row of this thread
    const int pos = p0 + r / G, hh = r % G;
    const bool row_valid = pos < Qb;
    const int limit = L - Qb + min(pos, Qb - 1);  // last key this row may see
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(bar(pf::B_SFULL + (j & 1)), (j >> 1) & 1))) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      const uint32_t sa = tmem + lane_off + (j & 1) * pf::S_BUF_COLS;
      uint32_t sr[pf::BN];
#pragma unroll
      for (int c = 0; c < pf::BN; c += 32) tc::ld_32x32b_x32(sa + c, sr + c);
      tc::wait_ld();
      const int kv0 = j * pf::BN;
      const bool diag = kv0 + pf::BN - 1 > limit;
      float mx = -INFINITY;
      if (diag) {
#pragma unroll
        for (int c = 0; c < pf::BN; ++c)
          if (kv0 + c <= limit) mx = fmaxf(mx, __uint_as_float(sr[c]));
      } else {
#pragma unroll
        for (int c = 0; c < pf::BN; ++c) mx = fmaxf(mx, __uint_as_float(sr[c]));
      }
      const float m_tile = (mx == -INFINITY) ? -INFINITY : mx * sl2;
      const bool grow = m_tile > m_run + pf::RESCALE_THRESHOLD;  // always true on the first tile
      if (__any_sync(0xffffffffu, grow)) {
        // warp-uniform branch: the TMEM accesses below are warp-collective;
        // rows that keep their max use alpha = 1
        const float alpha = grow ? ex2(m_run - m_tile) : 1.f;  // 0 on the first tile
        if (j > 0) {
          // O holds P.V of earlier tiles: rescale it once the last of them is done
          if (!__all_sync(0xffffffffu, mbar_wait(bar(pf::B_OREADY), (j - 1) & 1))) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint32_t oa = tmem + lane_off + pf::O_COL;
#pragma unroll
          for (int c = 0; c < pf::D; c += 32) {
            uint32_t o[32];
            tc::ld_32x32b_x32(oa + c, o);
            tc::wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tc::st_32x32b_x32(oa + c, o);
          }
          tc::wait_st();
        }
        if (grow) {
          l_run *= alpha;
          m_run = m_tile;
        }
      }
      // P = 2^(s * scale_log2 - m) as bf16 pairs, written over the score buffer
      float rs = 0.f;
      uint32_t pw[pf::BN / 2];
#pragma unroll
      for (int c = 0; c < pf::BN; c += 2) {
        float p0v = ex2(fmaf(__uint_as_float(sr[c]), sl2, -m_run));
        float p1v = ex2(fmaf(__uint_as_float(sr[c + 1]), sl2, -m_run));
        if (diag) {
          if (kv0 + c > limit) p0v = 0.f;
          if (kv0 + c + 1 > limit) p1v = 0.f;
        }
        rs += p0v + p1v;
        __nv_bfloat162 h2 = __floats2bfloat162_rn(p0v, p1v);
        pw[c / 2] = *reinterpret_cast<uint32_t*>(&h2);
      }
      l_run += rs;
      tc::st_32x32b_x32(sa, pw);
      tc::st_32x32b_x32(sa + 32, pw + 32);
      tc::wait_st();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(pf::B_PFULL + (j & 1)));
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(bar(pf::B_OREADY), (n_tiles - 1) & 1))) {
      tc::fence_after_sync();
      const uint32_t oa = tmem + lane_off + pf::O_COL;
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      uint4* dst = reinterpret_cast<uint4*>(p.out + ((size_t)(qs + pos) * p.Hq + kvh * G + hh) * pf::D);
#pragma unroll
      for (int c = 0; c < pf::D; c += 32) {
        uint32_t o[32];
        tc::ld_32x32b_x32(oa + c, o);
        tc::wait_ld();
        if (row_valid) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(o[v * 8 + 2 * e]) * inv,
                                                        __uint_as_float(o[v * 8 + 2 * e + 1]) * inv);
              w[e] = *reinterpret_cast<uint32_t*>(&h2);
            }
            dst[c / 8 + v] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown --
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 2) {
    tc::fence_after_sync();
    tc::dealloc(tmem, pf::TMEM_COLS);
  }
}

}  // namespace pkv
