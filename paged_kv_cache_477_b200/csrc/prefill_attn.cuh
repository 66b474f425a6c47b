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
// B200 design (one CTA per SM, 12 warps):
//   * A CTA owns a task: two 128-row query tiles of one (sequence, kv head).
//     The G query heads of the kv head are packed into the rows (row =
//     position * G + head), so every K/V tile loaded feeds 256 query rows.
//     The last query tiles of a chunk see the most keys; they are launched
//     first so the shortest CTAs fill the last wave.
//   * Warp 0 (lanes 0-7) loads Q once and K/V tiles through separate K and V
//     rings with tiled TMA: each 16-key page of the paged cache is one
//     16 x 64-element box per head-dim half, landing in the 128-byte-swizzled
//     layout the MMA reads.  A page beyond the context is addressed out of
//     range, so TMA fills it with zeros.
//   * Warp 1 (one lane) issues tcgen05.mma in ping-pong order: for each key
//     tile j, O_0 += P_0 V_{j-1}, S_0 = Q_0 K_j^T, O_1 += P_1 V_{j-1},
//     S_1 = Q_1 K_j^T.  P is read straight from TMEM (bf16 written over the
//     score columns it came from); V is an MN-major shared-memory operand.
//     While one softmax warpgroup works on its tile the tensor core runs the
//     other tile's two MMAs.
//   * Warps 4-7 and 8-11 are the two softmax warpgroups (thread = TMEM lane =
//     query row): load a score row, mask on diagonal tiles only, keep the
//     running max and sum, write P back.  Part of the exponentials run on the
//     FMA pipe as a polynomial so the MUFU unit is not the limit.  O is
//     rescaled in TMEM only when the running max grows by more than 2^8
//     (exact after the final division by the row sum).  The same warps
//     finish with O / l to global memory.
//   * TMEM (512 columns): per query tile a 128-column score buffer and a
//     128-column O accumulator.
//   * Every mbarrier wait is bounded; on a timeout each role stops, in-flight
//     copies and MMAs are waited for, and TMEM is released.
#pragma once
#include "pkv_common.cuh"
#include "tcgen05.cuh"

namespace pkv {

struct PrefillParams {
  __nv_bfloat16* out;              // [sumQ][Hq][128]
  const int32_t* query_start_loc;  // [B+1]
  const int32_t* block_tables;     // [B][MB]
  const int32_t* context_lens;     // [B]
  int32_t B, Hq, Hkv, NB, MB, G, sumQ;
  int32_t nct;                     // tasks (query-tile pairs) per (sequence, kv head)
  int32_t window;                  // > 0: a query at p sees only keys p - window < j <= p
  float scale_log2;                // scale * log2(e), >= 0
};

namespace pf {
constexpr int BM = 128;                 // query rows per tile
constexpr int NQT = 2;                  // query tiles per CTA
constexpr int BN = 128;                 // keys per tile (8 pages)
constexpr int KSTAGES = 3;
constexpr int VSTAGES = 2;
constexpr int HALF_BYTES = 128 * 128;   // 128 rows x 64 bf16 (one 64-element head-dim half)
constexpr int PAGE_BOX_BYTES = 16 * 128;  // one page, one half
// barriers
constexpr int B_Q = 0;
constexpr int B_KFULL = 1;
constexpr int B_KEMPTY = B_KFULL + KSTAGES;
constexpr int B_VFULL = B_KEMPTY + KSTAGES;
constexpr int B_VEMPTY = B_VFULL + VSTAGES;
constexpr int B_SFULL = B_VEMPTY + VSTAGES;  // per query tile
constexpr int B_PFULL = B_SFULL + NQT;       // per query tile, 4 arrivals
constexpr int B_OREADY = B_PFULL + NQT;      // per query tile
constexpr int B_MMADONE = B_OREADY + NQT;
constexpr int NUM_BARS = B_MMADONE + 1;
constexpr int THREADS = 384;
constexpr int TMEM_COLS = 512;
constexpr int TILE_COLS = 256;  // query tile i: scores at i*256, O at i*256 + 128
constexpr int O_COL = 128;
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units: rescale O when the max grows by > 2^8
#ifndef PKV_PREFILL_POLY_EVERY
#define PKV_PREFILL_POLY_EVERY 0  // measured fastest on B200: MUFU for every exponential
#endif
// one column pair in POLY_PAIR_EVERY takes the FMA-pipe exp2 (0: none)
constexpr int POLY_PAIR_EVERY = PKV_PREFILL_POLY_EVERY;
__host__ __device__ constexpr bool poly_pair(int pair) {
  return POLY_PAIR_EVERY > 0 && pair % (POLY_PAIR_EVERY > 0 ? POLY_PAIR_EVERY : 1) == POLY_PAIR_EVERY - 1;
}
constexpr int REGS_LAUNCH = 168;    // 65536 / 384 rounded down to a multiple of 8
constexpr int REGS_LOW = 64;        // load / MMA / allocator warpgroup
constexpr int REGS_HIGH = 216;      // softmax warpgroups
static_assert(4 * REGS_LOW + 8 * REGS_HIGH <= 12 * REGS_LAUNCH, "register split must fit the launch");

// Shared-memory layout for head size D: tiles of D/64 swizzled 64-element
// halves (query tiles, then K stages, then V stages), then the barriers.
template <int D>
struct Layout {
  static_assert(D == 64 || D == 128, "head_dim");
  static constexpr int NH = D / 64;
  static constexpr int TILE_BYTES = NH * HALF_BYTES;
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + NQT * TILE_BYTES;
  static constexpr int V_OFF = K_OFF + KSTAGES * TILE_BYTES;
  static constexpr int BAR_OFF = V_OFF + VSTAGES * TILE_BYTES;
  static constexpr int TMEM_SLOT_OFF = BAR_OFF + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = TMEM_SLOT_OFF + 16 + 1024;  // + slack to align the base to 1 KB
};
}  // namespace pf

// Three-input maximum (one ALU instruction on sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// 2^x on the FMA pipe (Cody-Waite style): x = n + f with n = round(x) found by
// the 1.5 * 2^23 shifter, f in [-0.5, 0.5]; 2^f by a degree-3 polynomial
// fitted here for minimum relative error on that interval (max relative error
// 7.5e-5 in fp32, below bf16's 2^-9 rounding of P); n is added to the
// exponent field.  Inputs are clamped at -126 so n never underflows the
// exponent; callers zero masked entries themselves.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  const float2 lo = make_float2(-126.f, -126.f);
  x = make_float2(fmaxf(x.x, lo.x), fmaxf(x.y, lo.y));
  const float2 shifter = make_float2(12582912.f, 12582912.f);
  const float2 j = __fadd2_rn(x, shifter);            // low mantissa bits hold round(x)
  const float2 n = __fadd2_rn(j, make_float2(-shifter.x, -shifter.y));  // round(x), exact
  const float2 f = __fadd2_rn(x, make_float2(-n.x, -n.y));
  float2 p = __ffma2_rn(make_float2(0.05517098f, 0.05517098f), f, make_float2(0.24260971f, 0.24260971f));
  p = __ffma2_rn(p, f, make_float2(0.69326097f, 0.69326097f));
  p = __ffma2_rn(p, f, make_float2(0.99992818f, 0.99992818f));
  const uint32_t ex = __float_as_uint(j.x) << 23, ey = __float_as_uint(j.y) << 23;
  return make_float2(__uint_as_float(__float_as_uint(p.x) + ex), __uint_as_float(__float_as_uint(p.y) + ey));
}

// Task t of a launch: query-tile pair ct of sequence b, kv head kvh, in grid
// order (kv head fastest, then sequence, then the pairs last first).  Its
// rows see key tiles [j0, n) (n = 0: nothing to do; j0 > 0 only under a
// sliding window, where the earliest row's window starts).  Each role of
// the CTA computes it for itself (three cached loads) instead of keeping it
// live across the register split.
struct PrefillTask {
  int b, kvh, ct, qs, Qb, L, p0, n, j0;
};

template <bool WIN>
__device__ __forceinline__ PrefillTask prefill_task(const PrefillParams& p, int t) {
  PrefillTask k;
  const int per = p.B * p.Hkv;
  k.ct = p.nct - 1 - t / per;
  k.b = (t % per) / p.Hkv;
  k.kvh = t % p.Hkv;
  k.qs = __ldg(p.query_start_loc + k.b);
  k.Qb = __ldg(p.query_start_loc + k.b + 1) - k.qs;
  k.L = __ldg(p.context_lens + k.b);
  k.p0 = k.ct * pf::NQT * (pf::BM / p.G);
  k.n = 0;
  k.j0 = 0;
  if (k.Qb < 0 || k.L < k.Qb || k.L > p.MB * 16 || k.qs < 0 || k.qs + k.Qb > p.sumQ) {
    set_error(PKV_ERR_BOUNDS);
  } else if (k.p0 < k.Qb) {
    const int last_pos = min(k.p0 + pf::NQT * (pf::BM / p.G), k.Qb) - 1;
    const int kv_end = k.L - k.Qb + last_pos + 1;  // keys the last valid row can see
    k.n = (kv_end + pf::BN - 1) / pf::BN;
    if (WIN) {
      const int first_key = k.L - k.Qb + k.p0 - p.window + 1;  // the first row's window start
      k.j0 = first_key > 0 ? first_key / pf::BN : 0;
    }
  }
  return k;
}

// WIN: sliding window of p.window keys (a separate instantiation, so the
// plain causal kernel carries none of its per-row bounds).
template <int D, bool WIN>
__global__ void __launch_bounds__(pf::THREADS, 1)
    prefill_attn_kernel(const __grid_constant__ PrefillParams p, const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v) {
  using LY = pf::Layout<D>;
  extern __shared__ __align__(16) unsigned char smem_raw[];  // base aligned to 1 KB by hand below
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* sbase = smem_raw + (base - raw);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.G, PPT = pf::BM / G;  // query positions per tile
  const int t = (blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;  // this CTA's task

  __shared__ int s_flag;
  if (threadIdx.x == 0) {
    int f = *reinterpret_cast<volatile int*>(&g_error_word) == PKV_ERR_TIMEOUT;
    f |= prefill_task<WIN>(p, t).n == 0;  // nothing to do (or bad lengths, reported)
    s_flag = f;
  }
  __syncthreads();
  if (s_flag) return;

  auto bar = [&](int i) { return base + LY::BAR_OFF + 8u * i; };
  if (threadIdx.x == 0) {
    mbar_init(bar(pf::B_Q), 1);
    for (int s = 0; s < pf::KSTAGES; ++s) {
      mbar_init(bar(pf::B_KFULL + s), 1);
      mbar_init(bar(pf::B_KEMPTY + s), 1);
    }
    for (int s = 0; s < pf::VSTAGES; ++s) {
      mbar_init(bar(pf::B_VFULL + s), 1);
      mbar_init(bar(pf::B_VEMPTY + s), 1);
    }
    for (int i = 0; i < pf::NQT; ++i) {
      mbar_init(bar(pf::B_SFULL + i), 1);
      mbar_init(bar(pf::B_PFULL + i), 4);  // one arrival per softmax warp
      mbar_init(bar(pf::B_OREADY + i), 1);
    }
    mbar_init(bar(pf::B_MMADONE), 1);
    fence_barrier_init();
  }
  if (warp == 2) {
    tc::alloc(base + LY::TMEM_SLOT_OFF, pf::TMEM_COLS);
    tc::relinquish_alloc_permit();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sbase + LY::TMEM_SLOT_OFF);

  // Register split (per thread): the load/MMA warpgroup gives up registers to
  // the two softmax warpgroups.  4 x REGS_LOW + 8 x REGS_HIGH <= 12 x
  // REGS_LAUNCH, the block's own pool; the host refuses to launch a build whose
  // register count differs from REGS_LAUNCH.
  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(pf::REGS_LOW));
    if (warp == 0) {
      // ---------------------------------------------------------- TMA loads --
      if (lane == 0) {
        tc::prefetch_tensormap(&tm_q);
        tc::prefetch_tensormap(&tm_k);
        tc::prefetch_tensormap(&tm_v);
      }
      const PrefillTask k = prefill_task<WIN>(p, t);
      if (lane == 0) {
        mbar_arrive_expect_tx(bar(pf::B_Q), pf::NQT * LY::TILE_BYTES);
        for (int i = 0; i < pf::NQT; ++i) {
          const uint32_t qd = base + LY::Q_OFF + i * LY::TILE_BYTES;
          const int z = k.qs + k.p0 + i * PPT;
#pragma unroll
          for (int h = 0; h < LY::NH; ++h)
            tc::tma_load_3d(qd + h * pf::HALF_BYTES, &tm_q, 64 * h, k.kvh * G, z, bar(pf::B_Q));
        }
      }
      const int32_t* bt = p.block_tables + (size_t)k.b * p.MB;
      const int npages = (k.L + 15) / 16;
      int issued_k = 0, issued_v = 0;
      bool ok = true;
      for (int j = k.j0; j < k.n; ++j) {
        const int jl = j - k.j0;  // position in this task's key-tile stream
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
        // K tile j
        const int ks = jl % pf::KSTAGES;
        if (lane == 0) {
          if (jl >= pf::KSTAGES) ok = mbar_wait(bar(pf::B_KEMPTY + ks), ((jl / pf::KSTAGES) - 1) & 1);
          if (ok) mbar_arrive_expect_tx(bar(pf::B_KFULL + ks), LY::TILE_BYTES);
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        if (lane < 8) {
          const uint32_t kd = base + LY::K_OFF + ks * LY::TILE_BYTES + lane * pf::PAGE_BOX_BYTES;
#pragma unroll
          for (int h = 0; h < LY::NH; ++h)
            tc::tma_load_4d(kd + h * pf::HALF_BYTES, &tm_k, 64 * h, 0, k.kvh, blk, bar(pf::B_KFULL + ks));
        }
        ++issued_k;
        // V tile j
        const int vs = jl % pf::VSTAGES;
        if (lane == 0) {
          if (jl >= pf::VSTAGES) ok = mbar_wait(bar(pf::B_VEMPTY + vs), ((jl / pf::VSTAGES) - 1) & 1);
          if (ok) mbar_arrive_expect_tx(bar(pf::B_VFULL + vs), LY::TILE_BYTES);
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        if (lane < 8) {
          const uint32_t vd = base + LY::V_OFF + vs * LY::TILE_BYTES + lane * pf::PAGE_BOX_BYTES;
#pragma unroll
          for (int h = 0; h < LY::NH; ++h)
            tc::tma_load_4d(vd + h * pf::HALF_BYTES, &tm_v, 64 * h, 0, k.kvh, blk, bar(pf::B_VFULL + vs));
        }
        ++issued_v;
      }
      // leave no copy in flight: wait for the last issued use of every buffer
      if (lane == 0) {
        mbar_wait(bar(pf::B_Q), 0);
        for (int s = 0; s < pf::KSTAGES && s < issued_k; ++s) {
          const int last = s + ((issued_k - 1 - s) / pf::KSTAGES) * pf::KSTAGES;
          mbar_wait(bar(pf::B_KFULL + s), (last / pf::KSTAGES) & 1);
        }
        for (int s = 0; s < pf::VSTAGES && s < issued_v; ++s) {
          const int last = s + ((issued_v - 1 - s) / pf::VSTAGES) * pf::VSTAGES;
          mbar_wait(bar(pf::B_VFULL + s), (last / pf::VSTAGES) & 1);
        }
      }
    } else if (warp == 1 && lane == 0) {
      // ------------------------------------------------------------- MMA ------
      // One thread: it alone waits on the barriers it needs and issues every
      // MMA and commit, so no warp-wide vote sits between two MMA groups.
      constexpr uint32_t IDESC_S = tc::idesc_bf16_f32(pf::BM, pf::BN, false, false);
      constexpr uint32_t IDESC_PV = tc::idesc_bf16_f32(pf::BM, D, false, true);
      // Descriptors are built once; a K step only moves the start address,
      // whose 14-bit field (address >> 4) cannot carry: shared memory < 256 KB.
      const uint64_t desc_q = tc::smem_desc_sw128(base + LY::Q_OFF, 16, 1024);
      const uint64_t desc_k = tc::smem_desc_sw128(base + LY::K_OFF, 16, 1024);
      const uint64_t desc_v = tc::smem_desc_sw128(base + LY::V_OFF, pf::HALF_BYTES, 1024);
      constexpr uint32_t TILE16 = LY::TILE_BYTES >> 4;
      int tk = 0, tv = 0;  // K and V tiles consumed: ring stage and phase
      auto qk = [&](int i) {  // S_i = Q_i K^T for K tile tk
        const int ks = tk % pf::KSTAGES;
        const uint64_t dq = desc_q + i * TILE16, dk = desc_k + ks * TILE16;
        const uint32_t d_s = tmem + i * pf::TILE_COLS;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off16 = ((kk >> 2) * pf::HALF_BYTES + (kk & 3) * 32) >> 4;
          tc::mma_ss(d_s, dq + off16, dk + off16, IDESC_S, kk > 0 ? 1u : 0u);
        }
        tc::commit(bar(pf::B_SFULL + i));
        if (i == pf::NQT - 1) tc::commit(bar(pf::B_KEMPTY + ks));
      };
      // O_i += P_i V for V tile tv = key tile j, the task's jl-th
      auto pv = [&](int i, int jl, int j, int tail_rows, int tail_page) -> bool {
        const int vs = tv % pf::VSTAGES;
        if (!mbar_wait(bar(pf::B_PFULL + i), jl & 1)) return false;
        if (i == 0) {
          if (!mbar_wait(bar(pf::B_VFULL + vs), (tv / pf::VSTAGES) & 1)) return false;
          if (tail_rows != 0 && tail_page / 8 == j) {
            // rows past the end of the context hold stale data that a zero
            // probability would not cancel if it were NaN: clear them
            unsigned char* vp = sbase + LY::V_OFF + vs * LY::TILE_BYTES + (tail_page % 8) * pf::PAGE_BOX_BYTES;
            const int nvec = (16 - tail_rows) * 8;  // 16-byte vectors per half
            for (int e = 0; e < LY::NH * nvec; ++e) {
              const int half = e / nvec, k = e % nvec;
              *reinterpret_cast<uint4*>(vp + half * pf::HALF_BYTES + tail_rows * 128 + k * 16) =
                  make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
          }
        }
        tc::fence_after_sync();
        const uint64_t dv = desc_v + vs * TILE16;
        const uint32_t p_t = tmem + i * pf::TILE_COLS;
        const uint32_t d_o = p_t + pf::O_COL;
#pragma unroll
        for (int kk = 0; kk < pf::BN / 16; ++kk)
          tc::mma_ts(d_o, p_t + kk * 8, dv + kk * (2048 >> 4), IDESC_PV, (jl > 0 || kk > 0) ? 1u : 0u);
        tc::commit(bar(pf::B_OREADY + i));
        if (i == pf::NQT - 1) {
          tc::commit(bar(pf::B_VEMPTY + vs));
          ++tv;
        }
        return true;
      };

      const PrefillTask k = prefill_task<WIN>(p, t);
      // the page holding the sequence's last key, if it is only partly valid
      const int tail_rows = k.L % 16, tail_page = (k.L - 1) / 16;
      bool ok = mbar_wait(bar(pf::B_Q), 0);
      if (ok) ok = mbar_wait(bar(pf::B_KFULL), 0);
      if (ok) {
        tc::fence_after_sync();
        for (int i = 0; i < pf::NQT; ++i) qk(i);
        ++tk;
      }
      const int nl = k.n - k.j0;  // key tiles of this task
      for (int jl = 1; jl < nl && ok; ++jl) {
        for (int i = 0; i < pf::NQT && ok; ++i) {
          ok = pv(i, jl - 1, k.j0 + jl - 1, tail_rows, tail_page);  // frees query tile i's score buffer
          if (ok && i == 0) ok = mbar_wait(bar(pf::B_KFULL + tk % pf::KSTAGES), (tk / pf::KSTAGES) & 1);
          if (ok) {
            tc::fence_after_sync();
            qk(i);
          }
        }
        ++tk;
      }
      for (int i = 0; i < pf::NQT && ok; ++i) ok = pv(i, nl - 1, k.n - 1, tail_rows, tail_page);
      // all MMAs of this CTA retired before TMEM is released
      tc::commit(bar(pf::B_MMADONE));
      mbar_wait(bar(pf::B_MMADONE), 0);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(pf::REGS_HIGH));
    // --------------------------------------------- softmax and epilogue -----
    const int qt = (warp - 4) >> 2;              // query tile of this warpgroup
    const int wq = warp & 3;                     // TMEM lane quarter of this warp
    const int r = wq * 32 + lane;                // row within the query tile
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t s_addr = tmem + lane_off + qt * pf::TILE_COLS;
    const uint32_t o_addr = s_addr + pf::O_COL;
    const float sl2 = p.scale_log2;
    const PrefillTask k = prefill_task<WIN>(p, t);
    const int pos = k.p0 + qt * PPT + r / G, hh = r % G;
    const bool row_valid = pos < k.Qb;
    const int limit = k.L - k.Qb + min(pos, k.Qb - 1);  // last key this row may see
    const int lo = WIN ? limit - p.window + 1 : 0;  // first key this row may see
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    {  // key tiles, then the epilogue
      for (int j = k.j0; j < k.n; ++j) {
        const int jl = j - k.j0;
        if (!__all_sync(0xffffffffu, mbar_wait(bar(pf::B_SFULL + qt), jl & 1))) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        uint32_t sr[pf::BN];
#pragma unroll
        for (int c = 0; c < pf::BN; c += 32) tc::ld_32x32b_x32(s_addr + c, sr + c);
        tc::wait_ld();
        const int kv0 = j * pf::BN;
        // edge tiles: the causal diagonal, or (sliding window) the row's window start
        const bool diag = kv0 + pf::BN - 1 > limit || (WIN && kv0 < lo);
        if (diag) {
#pragma unroll
          for (int c = 0; c < pf::BN; ++c)
            if (kv0 + c > limit || (WIN && kv0 + c < lo)) sr[c] = __float_as_uint(-INFINITY);
        }
        // row max: eight independent chains of three-input maxima
        float mxk[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          float m = fmax3(__uint_as_float(sr[16 * k]), __uint_as_float(sr[16 * k + 1]),
                          __uint_as_float(sr[16 * k + 2]));
#pragma unroll
          for (int e = 3; e < 15; e += 2)
            m = fmax3(m, __uint_as_float(sr[16 * k + e]), __uint_as_float(sr[16 * k + e + 1]));
          mxk[k] = fmaxf(m, __uint_as_float(sr[16 * k + 15]));
        }
        const float mx = fmax3(fmax3(mxk[0], mxk[1], mxk[2]), fmax3(mxk[3], mxk[4], mxk[5]), fmaxf(mxk[6], mxk[7]));
        const float m_tile = (mx == -INFINITY) ? -INFINITY : mx * sl2;
        const bool grow = m_tile > m_run + pf::RESCALE_THRESHOLD;  // always true on the first tile
        if (__any_sync(0xffffffffu, grow)) {
          // warp-uniform branch: the TMEM accesses below are warp-collective;
          // rows that keep their max use alpha = 1
          const float alpha = grow ? ex2(m_run - m_tile) : 1.f;  // 0 on the first tile
          if (jl > 0) {
            // O holds P.V of earlier tiles: rescale it once the last of them is done
            if (!__all_sync(0xffffffffu, mbar_wait(bar(pf::B_OREADY + qt), (jl - 1) & 1))) {
              ok = false;
              break;
            }
            tc::fence_after_sync();
#pragma unroll
            for (int c = 0; c < D; c += 32) {
              uint32_t o[32];
              tc::ld_32x32b_x32(o_addr + c, o);
              tc::wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              tc::st_32x32b_x32(o_addr + c, o);
            }
            tc::wait_st();
          }
          if (grow) {
            l_run *= alpha;
            m_run = m_tile;
          }
        }
        // P = 2^(s * scale_log2 - m) as bf16 pairs, written over the score
        // columns in two halves so the first store overlaps the second half
        const float2 sl2x2 = make_float2(sl2, sl2), negm = make_float2(-m_run, -m_run);
        float2 rs[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                        make_float2(0.f, 0.f)};
        uint32_t* pw = sr;  // packed P overwrites the scores already consumed (c/2 < c)
#pragma unroll
        for (int half = 0; half < 2; ++half) {
#pragma unroll
          for (int c = half * 64; c < half * 64 + 64; c += 2) {
            const float2 x =
                __ffma2_rn(make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sl2x2, negm);
            float2 pr = pf::poly_pair(c / 2)
                            ? exp2_poly2(x)
                            : make_float2(ex2(x.x), ex2(x.y));
            if (diag) {  // masked keys: exactly 0 (the polynomial, or a zero scale, would not give it)
              if (kv0 + c > limit || (WIN && kv0 + c < lo)) pr.x = 0.f;
              if (kv0 + c + 1 > limit || (WIN && kv0 + c + 1 < lo)) pr.y = 0.f;
            }
            rs[(c / 2) & 3] = __fadd2_rn(rs[(c / 2) & 3], pr);
            __nv_bfloat162 h2 = __floats2bfloat162_rn(pr.x, pr.y);
            pw[c / 2] = *reinterpret_cast<uint32_t*>(&h2);
          }
          tc::st_32x32b_x32(s_addr + half * 32, pw + half * 32);
        }
        const float2 r01 = __fadd2_rn(rs[0], rs[1]), r23 = __fadd2_rn(rs[2], rs[3]);
        const float2 rr = __fadd2_rn(r01, r23);
        l_run += rr.x + rr.y;
        tc::wait_st();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(pf::B_PFULL + qt));
      }
      if (ok && __all_sync(0xffffffffu, mbar_wait(bar(pf::B_OREADY + qt), (k.n - k.j0 - 1) & 1))) {
        tc::fence_after_sync();
        uint4* dst = reinterpret_cast<uint4*>(p.out + ((size_t)(k.qs + pos) * p.Hq + k.kvh * G + hh) * D);
        // O / l to global memory
        const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t o[32];
          tc::ld_32x32b_x32(o_addr + c, o);
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
