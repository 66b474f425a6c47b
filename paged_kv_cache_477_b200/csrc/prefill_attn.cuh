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
//     position * G + head), so every K/V tile loaded feeds 256 query rows;
//     a tile holds floor(128 / G) whole positions (when G does not divide
//     128 its last rows stay idle).
//     The tasks of one (sequence, kv head) are consecutive in the grid, so
//     they run in the same wave and its K/V pages cross HBM once.
//   * Warp 0 (lanes 0-7) loads Q once and the K tiles of 128 keys (eight
//     16-key pages), warp 3 the V tiles, through separate rings with tiled
//     TMA: each page is one 16 x 64-element box per head-dim half, landing in
//     the 128-byte-swizzled layout the MMA reads.  A page beyond the context
//     is addressed out of range, so TMA fills it with zeros.
//   * TMEM (512 columns): one 128-column score buffer S shared by the two
//     query tiles, a 64-column bf16 P buffer per query tile, and a D-column
//     O accumulator per query tile.  A softmax warpgroup hands S back as soon
//     as it has loaded it into registers, so the next Q.K^T (of the other
//     query tile) runs on the tensor core while this warpgroup computes its
//     exponentials; P goes to the tile's own P buffer, read by O += P V.
//   * Two threads issue tcgen05.mma, each alone on its warp.  Warp 1 issues
//     the scores in this order: S_1(j) = Q_1 K(j)^T once warpgroup 0 has
//     taken S_0(j), S_0(j+1) once warpgroup 1 has taken S_1(j); the two
//     warpgroups thus run half a step apart, each finding its next scores
//     ready when it finishes a tile.  Warp 2 issues O_i += P_i(j) V(j) as
//     each P arrives.  A barrier wait in an issuing thread stalls its own
//     stream only, so the tensor core is fed by the other one meanwhile.
//   * Warps 4-7 and 8-11 are the two softmax warpgroups, one per query tile
//     (thread = TMEM lane = query row): load a score row, mask on edge tiles
//     only, keep the running max and sum, write P.  O is rescaled in TMEM
//     only when the running max grows by more than 2^8 (exact after the final
//     division by the row sum).  The same warps finish with O / l to global
//     memory.
//   * A negative scale reverses the order of the scores: the row maximum of
//     scale * s is then scale times the row minimum of s.
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
  float scale_log2;                // scale * log2(e), finite, any sign
};

namespace pf {
constexpr int BM = 128;                 // query rows per tile
constexpr int NQT = 2;                  // query tiles per CTA
constexpr int BN = 128;                 // keys per tile (8 pages)
constexpr int PAGES = BN / 16;          // pages per key tile
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
constexpr int B_SFULL = B_VEMPTY + VSTAGES;  // per query tile: its scores are in S
constexpr int B_SFREE = B_SFULL + NQT;       // per query tile, 4 arrivals: its scores left S
constexpr int B_PFULL = B_SFREE + NQT;       // per query tile, 4 arrivals: P written
constexpr int B_OREADY = B_PFULL + NQT;      // per query tile: O += P V done (P buffer free)
constexpr int B_SDONE = B_OREADY + NQT;      // every Q.K^T MMA retired
constexpr int B_PVDONE = B_SDONE + 1;        // every P.V MMA retired
constexpr int B_DONE = B_PVDONE + 1;         // every role is done with TMEM: 8 softmax warps, 2 MMA issuers, 2 loaders
constexpr int DONE_ARRIVALS = 12;
constexpr int NUM_BARS = B_DONE + 1;
constexpr int THREADS = 384;
constexpr int TMEM_COLS = 512;
constexpr int S_COL = 0;                // shared score buffer, 128 columns
constexpr int P_COL = 128;              // query tile i: P at 128 + 64 i (bf16 pairs)
constexpr int O_COL = 256;              // query tile i: O at 256 + 128 i
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units: rescale O when the max grows by > 2^8
// One column pair in poly_every<D>() takes the FMA-pipe exp2 instead of the
// MUFU one (0: none).  Measured on B200: at head size 64 one pair in eight
// (507-512 vs 499 TFLOP/s: the exponentials weigh twice as much against MMAs
// half as long); at 128 none (one in eight: no change, one in four: 1.4 %
// slower, one in two: 6 % slower).  PKV_PREFILL_POLY_EVERY overrides both.
template <int D>
__host__ __device__ constexpr int poly_every() {
#ifdef PKV_PREFILL_POLY_EVERY
  return PKV_PREFILL_POLY_EVERY;
#else
  return D == 64 ? 8 : 0;
#endif
}
template <int D>
__host__ __device__ constexpr bool poly_pair(int pair) {
  return poly_every<D>() > 0 && pair % (poly_every<D>() > 0 ? poly_every<D>() : 1) == poly_every<D>() - 1;
}
constexpr int REGS_LAUNCH = 168;    // 65536 / 384 rounded down to a multiple of 8
// setmaxnreg takes one count per warpgroup: every warp of a warpgroup must
// execute the same instruction with the same count
constexpr int REGS_LOW = 72;        // load / MMA / allocator warpgroup
constexpr int REGS_HIGH = 216;      // softmax warpgroups
static_assert(4 * REGS_LOW + 8 * REGS_HIGH <= 12 * REGS_LAUNCH, "register split must fit the launch");
static_assert(O_COL + NQT * 128 <= TMEM_COLS && P_COL + NQT * BN / 2 <= O_COL, "TMEM columns");

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

// Three-input maximum and minimum (one ALU instruction each on sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float fmin3(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// 2^x on the FMA pipe (Cody-Waite style): x = n + f with n = round(x) found by
// the 1.5 * 2^23 shifter, f in [-0.5, 0.5]; 2^f by a degree-3 polynomial
// fitted here for minimum relative error on that interval (max relative error
// 7.5e-5 in fp32, below bf16's 2^-9 rounding of P); n is added to the
// exponent field.  Inputs are clamped at -126 so n never underflows the
// exponent; callers zero masked entries themselves.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  x = make_float2(fmaxf(x.x, -126.f), fmaxf(x.y, -126.f));
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

// One level of a tree of three-input extrema over the first W values of v,
// then the next level (constant trip counts, so v stays in registers).
template <bool MAX, int W>
__device__ __forceinline__ void fold3(float* v) {
  if constexpr (W > 1) {
    constexpr int NW = (W + 2) / 3;
#pragma unroll
    for (int k = 0; k < NW; ++k) {
      const float a = v[3 * k];
      const float b = 3 * k + 1 < W ? v[3 * k + 1] : a;
      const float c = 3 * k + 2 < W ? v[3 * k + 2] : a;
      v[k] = MAX ? fmax3(a, b, c) : fmin3(a, b, c);
    }
    fold3<MAX, NW>(v);
  }
}

// Largest (MAX) or smallest value of N scores: N/16 independent chains of
// three-input extrema, folded three at a time.  (A full tree of depth log3 N
// measured no faster on B200.)
template <bool MAX, int N>
__device__ __forceinline__ float row_extreme(const uint32_t* sr) {
  auto e3 = [](float a, float b, float c) { return MAX ? fmax3(a, b, c) : fmin3(a, b, c); };
  auto e2 = [](float a, float b) { return MAX ? fmaxf(a, b) : fminf(a, b); };
  constexpr int NC = N / 16;
  float ch[NC];
#pragma unroll
  for (int k = 0; k < NC; ++k) {
    float m = e3(__uint_as_float(sr[16 * k]), __uint_as_float(sr[16 * k + 1]), __uint_as_float(sr[16 * k + 2]));
#pragma unroll
    for (int e = 3; e < 15; e += 2) m = e3(m, __uint_as_float(sr[16 * k + e]), __uint_as_float(sr[16 * k + e + 1]));
    ch[k] = e2(m, __uint_as_float(sr[16 * k + 15]));
  }
  fold3<MAX, NC>(ch);
  return ch[0];
}

// The task of this CTA: query-tile pair ct of sequence b, kv head kvh.  The
// grid is (pairs, kv heads, sequences) with the pairs fastest, so the tasks
// of one (sequence, kv head) are launched together, its last pair first.
// The task's rows see key tiles [j0, n) (n = 0: nothing to do; j0 > 0 only
// under a sliding window, where the earliest row's window starts).  Each role
// of the CTA computes it for itself (three cached loads) instead of keeping it
// live across the register split.
struct PrefillTask {
  int b, kvh, ct, qs, Qb, L, p0, n, j0;
};

template <bool WIN>
__device__ __forceinline__ PrefillTask prefill_task(const PrefillParams& p) {
  PrefillTask k;
  k.ct = p.nct - 1 - (int)blockIdx.x;
  k.kvh = blockIdx.y;
  k.b = blockIdx.z;
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

  __shared__ int s_flag;
  if (threadIdx.x == 0) {
    int f = *reinterpret_cast<volatile int*>(&g_error_word) == PKV_ERR_TIMEOUT;
    f |= prefill_task<WIN>(p).n == 0;  // nothing to do (or bad lengths, reported)
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
      mbar_init(bar(pf::B_SFREE + i), 4);  // one arrival per softmax warp
      mbar_init(bar(pf::B_PFULL + i), 4);
      mbar_init(bar(pf::B_OREADY + i), 1);
    }
    mbar_init(bar(pf::B_SDONE), 1);
    mbar_init(bar(pf::B_PVDONE), 1);
    mbar_init(bar(pf::B_DONE), pf::DONE_ARRIVALS);
    fence_barrier_init();
  }
  if (warp == 4) {  // softmax warp 4 owns the TMEM allocation (all its lanes stay to free it)
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
    if (warp == 0 || warp == 3) {
      // ---------------------------------------------------------- TMA loads --
      // Warp 0 loads Q and the K tiles, warp 3 the V tiles: the two rings run
      // independently, so K(j+1), needed half a step before V(j), is never
      // queued behind a V copy waiting for its stage.
      const bool kload = warp == 0;
      const CUtensorMap* tm = kload ? &tm_k : &tm_v;
      const int nst = kload ? pf::KSTAGES : pf::VSTAGES;
      const int full0 = kload ? pf::B_KFULL : pf::B_VFULL, empty0 = kload ? pf::B_KEMPTY : pf::B_VEMPTY;
      const uint32_t ring = base + (kload ? LY::K_OFF : LY::V_OFF);
      if (lane == 0) {
        if (kload) tc::prefetch_tensormap(&tm_q);
        tc::prefetch_tensormap(tm);
      }
      const PrefillTask k = prefill_task<WIN>(p);
      if (kload && lane == 0) {
        // a query tile holds PPT whole positions of G heads: G * PPT <= 128
        // rows (the rows past them are never loaded and never written out)
        mbar_arrive_expect_tx(bar(pf::B_Q), pf::NQT * LY::NH * 128 * G * PPT);
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
      int issued = 0;
      bool ok = true;
      for (int j = k.j0; j < k.n; ++j) {
        const int jl = j - k.j0;  // position in this task's key-tile stream
        int blk = p.NB;  // out of range: TMA fills the page with zeros
        if (lane < pf::PAGES) {
          const int pg = j * pf::PAGES + lane;
          if (pg < npages) {
            blk = __ldg(bt + pg);
            if (blk < 0 || blk >= p.NB) {
              if (kload) set_error(PKV_ERR_BOUNDS);
              blk = p.NB;
            }
          }
        }
        const int st = jl % nst;
        if (lane == 0) {
          if (jl >= nst) ok = mbar_wait(bar(empty0 + st), ((jl / nst) - 1) & 1);
          if (ok) mbar_arrive_expect_tx(bar(full0 + st), LY::TILE_BYTES);
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        if (lane < pf::PAGES) {
          const uint32_t d = ring + st * LY::TILE_BYTES + lane * pf::PAGE_BOX_BYTES;
#pragma unroll
          for (int h = 0; h < LY::NH; ++h) tc::tma_load_4d(d + h * pf::HALF_BYTES, tm, 64 * h, 0, k.kvh, blk, bar(full0 + st));
        }
        ++issued;
      }
      // leave no copy in flight: wait for the last issued use of every stage
      if (lane == 0) {
        if (kload) mbar_wait(bar(pf::B_Q), 0);
        for (int s = 0; s < nst && s < issued; ++s) {
          const int last = s + ((issued - 1 - s) / nst) * nst;
          mbar_wait(bar(full0 + s), (last / nst) & 1);
        }
        mbar_arrive(bar(pf::B_DONE));
      }
    } else if ((warp == 1 || warp == 2) && lane == 0) {
      // ------------------------------------------------------------- MMA ------
      // Two issuing threads, each alone on its warp: warp 1 issues every
      // S = Q K^T, warp 2 every O += P V.  A barrier wait in an issuing thread
      // leaves the tensor core without new work while it lasts; with two
      // streams, one thread's waits are covered by the other's MMAs.
      const PrefillTask k = prefill_task<WIN>(p);
      const int nl = k.n - k.j0;  // key tiles of this task
      constexpr uint32_t TILE16 = LY::TILE_BYTES >> 4;
      bool ok = true;
      if (warp == 1) {
        constexpr uint32_t IDESC_S = tc::idesc_bf16_f32(pf::BM, pf::BN, false, false);
        // Descriptors are built once; a K step only moves the start address,
        // whose 14-bit field (address >> 4) cannot carry: shared memory < 256 KB.
        const uint64_t desc_q = tc::smem_desc_sw128(base + LY::Q_OFF, 16, 1024);
        const uint64_t desc_k = tc::smem_desc_sw128(base + LY::K_OFF, 16, 1024);
        // S = Q_i K(jl)^T into the shared score buffer
        auto qk = [&](int i, int jl) {
          const int ks = jl % pf::KSTAGES;
          const uint64_t dq = desc_q + i * TILE16, dk = desc_k + ks * TILE16;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off16 = ((kk >> 2) * pf::HALF_BYTES + (kk & 3) * 32) >> 4;
            tc::mma_ss(tmem + pf::S_COL, dq + off16, dk + off16, IDESC_S, kk > 0 ? 1u : 0u);
          }
          tc::commit(bar(pf::B_SFULL + i));
          if (i == pf::NQT - 1) tc::commit(bar(pf::B_KEMPTY + ks));
        };
        ok = mbar_wait(bar(pf::B_Q), 0) && mbar_wait(bar(pf::B_KFULL), 0);
        if (ok) {
          tc::fence_after_sync();
          qk(0, 0);
        }
        // Step jl, half h: once warpgroup h has taken its scores S_h(jl) out
        // of the score buffer, the other tile's next scores go in: S_1(jl)
        // for h = 0, S_0(jl+1) for h = 1.
        for (int jl = 0; jl < nl && ok; ++jl) {
          for (int h = 0; h < pf::NQT && ok; ++h) {
            const int js = jl + h;  // key tile of the scores issued now
            if (js >= nl) break;
            ok = mbar_wait(bar(pf::B_SFREE + h), jl & 1);
            if (ok && h == 1) ok = mbar_wait(bar(pf::B_KFULL + js % pf::KSTAGES), (js / pf::KSTAGES) & 1);
            if (ok) {
              tc::fence_after_sync();
              qk(1 - h, js);
            }
          }
        }
        tc::commit(bar(pf::B_SDONE));
        mbar_wait(bar(pf::B_SDONE), 0);
      } else {
        constexpr uint32_t IDESC_PV = tc::idesc_bf16_f32(pf::BM, D, false, true);
        const uint64_t desc_v = tc::smem_desc_sw128(base + LY::V_OFF, pf::HALF_BYTES, 1024);
        // the page holding the sequence's last key, if it is only partly valid
        const int tail_rows = k.L % 16, tail_page = (k.L - 1) / 16;
        for (int jl = 0; jl < nl && ok; ++jl) {
          const int vs = jl % pf::VSTAGES;
          for (int i = 0; i < pf::NQT && ok; ++i) {
            // O_i += P_i(jl) V(jl) for key tile j0 + jl
            ok = mbar_wait(bar(pf::B_PFULL + i), jl & 1);
            if (ok && i == 0) {
              ok = mbar_wait(bar(pf::B_VFULL + vs), (jl / pf::VSTAGES) & 1);
              if (ok && tail_rows != 0 && tail_page / pf::PAGES == k.j0 + jl) {
                // rows past the end of the context hold stale data that a zero
                // probability would not cancel if it were NaN: clear them
                const uint32_t vp = base + LY::V_OFF + vs * LY::TILE_BYTES +
                                    (tail_page % pf::PAGES) * pf::PAGE_BOX_BYTES + tail_rows * 128;
                const int nbytes = (16 - tail_rows) * 128;  // per half
#pragma unroll
                for (int half = 0; half < LY::NH; ++half)
                  for (int e = 0; e < nbytes; e += 16) st_shared_zero16(vp + half * pf::HALF_BYTES + e);
                fence_proxy_async_smem();
              }
            }
            if (!ok) break;
            tc::fence_after_sync();
            const uint64_t dv = desc_v + vs * TILE16;
            const uint32_t p_t = tmem + pf::P_COL + i * (pf::BN / 2);
            const uint32_t d_o = tmem + pf::O_COL + i * 128;
#pragma unroll
            for (int kk = 0; kk < pf::BN / 16; ++kk)
              tc::mma_ts(d_o, p_t + kk * 8, dv + kk * (2048 >> 4), IDESC_PV, (jl > 0 || kk > 0) ? 1u : 0u);
            tc::commit(bar(pf::B_OREADY + i));
            if (i == pf::NQT - 1) tc::commit(bar(pf::B_VEMPTY + vs));
          }
        }
        tc::commit(bar(pf::B_PVDONE));
        mbar_wait(bar(pf::B_PVDONE), 0);
      }
      // this thread's MMAs have retired before TMEM is released
      tc::fence_before_sync();
      mbar_arrive(bar(pf::B_DONE));
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(pf::REGS_HIGH));
    // --------------------------------------------- softmax and epilogue -----
    const int qt = (warp - 4) >> 2;              // query tile of this warpgroup
    const int wq = warp & 3;                     // TMEM lane quarter of this warp
    const int r = wq * 32 + lane;                // row within the query tile
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t s_addr = tmem + lane_off + pf::S_COL;
    const uint32_t p_addr = tmem + lane_off + pf::P_COL + qt * (pf::BN / 2);
    const uint32_t o_addr = tmem + lane_off + pf::O_COL + qt * 128;
    const float sl2 = p.scale_log2;
    // a negative scale turns the row minimum of the raw scores into the row
    // maximum of the scaled ones; masked scores take the value no extreme picks
    const bool neg = sl2 < 0.f;
    const uint32_t masked_bits = __float_as_uint(neg ? INFINITY : -INFINITY);
    const PrefillTask k = prefill_task<WIN>(p);
    const int pos = k.p0 + qt * PPT + r / G, hh = r % G;
    const bool row_valid = r < PPT * G && pos < k.Qb;
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
        // the scores are in registers: the score buffer is free for the other tile
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(pf::B_SFREE + qt));
        const int kv0 = j * pf::BN;
        // edge tiles: the causal diagonal, or (sliding window) the row's window start
        const bool diag = kv0 + pf::BN - 1 > limit || (WIN && kv0 < lo);
        if (diag) {
#pragma unroll
          for (int c = 0; c < pf::BN; ++c)
            if (kv0 + c > limit || (WIN && kv0 + c < lo)) sr[c] = masked_bits;
        }
        const float ext = neg ? row_extreme<false, pf::BN>(sr) : row_extreme<true, pf::BN>(sr);
        const float m_tile = (__float_as_uint(ext) == masked_bits) ? -INFINITY : ext * sl2;
        const bool grow = m_tile > m_run + pf::RESCALE_THRESHOLD;  // always true on the first tile
        // O += P(jl-1) V(jl-1) must be done before O is rescaled or the P
        // buffer is written again
        bool o_done = jl == 0;
        if (__any_sync(0xffffffffu, grow)) {
          // warp-uniform branch: the TMEM accesses below are warp-collective;
          // rows that keep their max use alpha = 1
          const float alpha = grow ? ex2(m_run - m_tile) : 1.f;  // 0 on the first tile
          if (jl > 0) {
            if (!__all_sync(0xffffffffu, mbar_wait(bar(pf::B_OREADY + qt), (jl - 1) & 1))) {
              ok = false;
              break;
            }
            o_done = true;
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
        // P = 2^(s * scale_log2 - m) as bf16 pairs
        const float2 sl2x2 = make_float2(sl2, sl2), negm = make_float2(-m_run, -m_run);
        float2 rs[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                        make_float2(0.f, 0.f)};
        uint32_t* pw = sr;  // packed P overwrites the scores already consumed (c/2 < c)
#pragma unroll
        for (int c = 0; c < pf::BN; c += 2) {
          const float2 x =
              __ffma2_rn(make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sl2x2, negm);
          float2 pr = pf::poly_pair<D>(c / 2) ? exp2_poly2(x) : make_float2(ex2(x.x), ex2(x.y));
          if (diag) {  // masked keys: exactly 0 (the polynomial, or a zero scale, would not give it)
            if (kv0 + c > limit || (WIN && kv0 + c < lo)) pr.x = 0.f;
            if (kv0 + c + 1 > limit || (WIN && kv0 + c + 1 < lo)) pr.y = 0.f;
          }
          rs[(c / 2) & 3] = __fadd2_rn(rs[(c / 2) & 3], pr);
          __nv_bfloat162 h2 = __floats2bfloat162_rn(pr.x, pr.y);
          pw[c / 2] = *reinterpret_cast<uint32_t*>(&h2);
        }
        const float2 r01 = __fadd2_rn(rs[0], rs[1]), r23 = __fadd2_rn(rs[2], rs[3]);
        const float2 rr = __fadd2_rn(r01, r23);
        l_run += rr.x + rr.y;
        if (!o_done) {
          if (!__all_sync(0xffffffffu, mbar_wait(bar(pf::B_OREADY + qt), (jl - 1) & 1))) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
        }
#pragma unroll
        for (int c = 0; c < pf::BN / 2; c += 32) tc::st_32x32b_x32(p_addr + c, pw + c);
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
    tc::fence_before_sync();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(pf::B_DONE));
  }

  // ------------------------------------------------------------ teardown --
  // Each role arrives on B_DONE once its MMAs, copies and TMEM accesses are
  // over, and warp 4, which allocated TMEM, frees it after the last arrival.
  // There is no CTA-wide barrier: the idle lanes of the MMA warps leave at
  // once instead of waiting at a barrier beside the lanes issuing MMAs.
  if (warp == 4) {
    mbar_wait(bar(pf::B_DONE), 0);
    __syncwarp();
    tc::fence_after_sync();
    tc::dealloc(tmem, pf::TMEM_COLS);
  }
}

}  // namespace pkv
