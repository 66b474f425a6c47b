// decode_attn_i8.cuh -- decode attention over the INT8 KV cache with the
// scores on the tensor cores.
//
// The INT8 cache (Tiny-Infer page, section "推测性解码与INT8量化": INT8 keys
// and values at half the memory of FP16) stores each (token, kv head) row as
// int8 codes with one fp32 scale.  Read by CUDA cores, turning codes into
// floats costs more instructions than the bf16 kernel spends per row, so the
// kernel would be bound by instruction issue at about the bf16 speed.  Here
// the codes never become floats on the K side:
//
//   S[key][n] = sum_d code_k[key][d] * Qi[n][d]           (tcgen05.mma kind::i8)
//
// with the query held as integers: per head h a power of two 2^e_h puts q into
// [-2^14, 2^14] (exact for every element within 2^7 of the head's largest;
// smaller ones are rounded to 2^-e_h), split into two signed bytes
// qi = 256 hi + lo.  Rows hi (n = h) and lo (n = HG + h) of the MMA's B
// operand give the exact integer q.k as 256 S_hi + S_lo in s32; the score is
// that integer times k_scale * scale * log2(e) * 2^-e_h.  V stays on the CUDA
// cores (the probabilities are fp32).
//
// One CTA per (split, head group, sequence): 4 consumer warps and two loader
// warps, one loading K and issuing the MMAs, one loading V and the row
// scales.  A tile is 8 pages = 128 keys (the MMA's M): their K codes arrive
// by tiled TMA into 128- (D=128) or 64-byte (D=64) swizzled rows, their V
// codes by 1-D bulk copies, their row scales by 16-byte cp.async from the
// second loader warp's lanes.  The MMA writes the tile's scores into one of
// two TMEM buffers (16 columns each); consumer warp w owns TMEM lanes
// 32w..32w+31, i.e. the tile's keys 32w..32w+31 (pages 2w, 2w+1), and keeps
// its own online-softmax state over them, merged across warps at the end as
// in the bf16 decode kernel.  Each lane first takes its own key's weights
// (one exp per key and head, V scale folded in); then the warp's lanes, 16
// elements of D each, accumulate the 32 rows of V codes with those weights.
#pragma once
#include <cuda.h>

#include "decode_attn.cuh"
#include "tcgen05.cuh"

namespace pkv {

template <int D, int HG>
struct DecodeI8Shape {
  static_assert(D == 64 || D == 128, "head_dim");
  static_assert(HG == 1 || HG == 2 || HG == 4, "heads per CTA");
  static constexpr int NW = 4;                    // consumer warps
  static constexpr int THREADS = (NW + 2) * 32;   // + a K/MMA warp and a V/scales warp
  static constexpr int TILE_PAGES = 8;
  static constexpr int TILE_ROWS = TILE_PAGES * kPageRows;  // 128 = MMA M
  static constexpr int WROWS = TILE_ROWS / NW;              // 32 keys per consumer warp
  static constexpr int PAGE = kPageRows * D;                // bytes of one page of codes
  static constexpr int ST = D == 128 ? 3 : 6;               // ring stages
  static constexpr int MMA_N = 16;                          // hi rows, lo rows, zero rows
  static constexpr int KSTEPS = D / 32;                     // 32 bytes of K per MMA
  static constexpr uint32_t SW_LAYOUT = D == 128 ? 2 : 4;   // 128- or 64-byte swizzle
  static constexpr int SBO = 8 * D;                         // bytes per 8-row swizzle atom
  static constexpr int TMEM_COLS = 32;                      // two score buffers
  // shared memory, offsets from a 1024-byte aligned base
  static constexpr int K_TILE = TILE_ROWS * D;              // 16 KB / 8 KB
  static constexpr int K_OFF = 0;
  static constexpr int Q_OFF = K_OFF + ST * K_TILE;
  static constexpr int Q_BYTES = MMA_N * D;
  static constexpr int V_OFF = Q_OFF + (Q_BYTES + 1023) / 1024 * 1024;
  static constexpr int SC_STAGE = 2 * TILE_ROWS * 4;        // K then V row scales of a tile
  static constexpr int S_OFF = V_OFF + ST * K_TILE;
  static constexpr int P_OFF = S_OFF + ST * SC_STAGE;       // scores [NW][WROWS][4] fp32
  static constexpr int BAR_OFF = P_OFF + NW * WROWS * 16;   // full[ST] empty[ST] sfull[2] sfree[2]
  static constexpr int MISC_OFF = BAR_OFF + (2 * ST + 4) * 8;  // TMEM base address, cq[4]
  static constexpr int SMEM_BYTES = MISC_OFF + 32 + 1024;      // + room to align the base
  // one warp's merge data, in the K ring after the last tile
  static constexpr int MERGE_STRIDE = (HG * D + 2 * HG + 3) / 4 * 4;
  static_assert(NW * MERGE_STRIDE * 4 <= ST * K_TILE, "merge data must fit the K ring");
  static_assert(K_TILE % 1024 == 0 && Q_OFF % 1024 == 0, "swizzled tiles start on 1024 bytes");
};

// Byte offset of element d of row r in a swizzled row-major tile of D-byte
// rows (the placement tiled TMA uses for 128- and 64-byte swizzle).
template <int D>
__device__ __forceinline__ int swizzled_offset(int r, int d) {
  const int chunk = d >> 4;
  const int x = D == 128 ? (r & 7) : ((r >> 1) & 3);
  return r * D + ((chunk ^ x) << 4) + (d & 15);
}

template <int D, int HG, bool WIN = false>
__global__ void __launch_bounds__(DecodeI8Shape<D, HG>::THREADS)
    decode_attn_i8_kernel(const __grid_constant__ DecodeParams p, const __grid_constant__ CUtensorMap tm_k) {
  using S = DecodeI8Shape<D, HG>;
  extern __shared__ __align__(128) unsigned char smem_i8[];
  const uint32_t raw_addr = smem_addr(smem_i8);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;  // swizzled tiles start on 1 KB
  unsigned char* sbase = smem_i8 + (base - raw_addr);

  const int split = blockIdx.x, hsub = blockIdx.y, b = blockIdx.z;
  const int kvh = hsub / p.nsub;
  const int head0 = kvh * p.G + (hsub % p.nsub) * HG;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool loader = warp >= S::NW;
  const int lid = warp - S::NW;          // 0: K codes by TMA and the MMAs; 1: V codes and row scales

  int L = __ldg(p.context_lens + b);
  const int wp0 = WIN ? window_first_key(L < 0 ? 0 : min(L, p.cap_tokens), p.window) / kPageRows : 0;
  const int pg0 = wp0 + split * p.pages_per_split;
  // block-table entries: lane l of chunk c holds the entry of the CTA's page
  // 32c + l; the first two chunks are loaded with the context length
  const int32_t* btrow = p.block_tables + (size_t)b * p.MB;
  auto load_raw = [&](int c) {
    const int w = c * 32 + lane;
    return (w < p.pages_per_split && pg0 + w < p.MB) ? __ldg(btrow + pg0 + w) : 0;
  };
  int ent_cur = 0, ent_nxt = 0;
  if (loader) {
    ent_cur = load_raw(0);
    ent_nxt = load_raw(1);
  }
  if (L < 0 || L > p.cap_tokens) {
    if (threadIdx.x == 0) set_error(PKV_ERR_BOUNDS);
    L = L < 0 ? 0 : p.cap_tokens;
  }
  const int npages = (L + kPageRows - 1) / kPageRows;
  const int n = min(npages - pg0, p.pages_per_split);  // pages of this CTA
  if (n <= 0) {  // a split past the sequence's end leaves at once; an empty context writes zeros
    if (p.num_splits == 1)
      for (int i = threadIdx.x; i < HG * D; i += blockDim.x)
        p.out[((size_t)b * p.Hq + head0 + i / D) * D + i % D] = __float2bfloat16_rn(0.f);
    return;
  }
  __shared__ int s_stop;
  if (threadIdx.x == 0) s_stop = *reinterpret_cast<volatile int*>(&g_error_word) == PKV_ERR_TIMEOUT;
  __syncthreads();
  if (s_stop) return;
  const int nt = (n + S::TILE_PAGES - 1) / S::TILE_PAGES;  // tiles of this CTA

  auto full = [&](int s) { return base + S::BAR_OFF + 8 * s; };
  auto empty = [&](int s) { return base + S::BAR_OFF + 8 * (S::ST + s); };
  auto sfull = [&](int i) { return base + S::BAR_OFF + 8 * (2 * S::ST + i); };
  auto sfree = [&](int i) { return base + S::BAR_OFF + 8 * (2 * S::ST + 2 + i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sbase + S::MISC_OFF);
  float* cq = reinterpret_cast<float*>(sbase + S::MISC_OFF + 16);  // per head: scale * log2(e) * 2^-e_h

  // ------------------------------------------------------------- set-up --
  if (loader && lid == 0) {
    if (lane == 0) {
      for (int s = 0; s < S::ST; ++s) {
        mbar_init(full(s), 2 + 32);  // each loader's bytes, then one per lane's row scales
        mbar_init(empty(s), S::NW);
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(sfull(i), 1);
        mbar_init(sfree(i), S::NW);
      }
      fence_barrier_init();
    }
    __syncwarp();
    tc::alloc(smem_addr(tmem_slot), S::TMEM_COLS);
    tc::relinquish_alloc_permit();
  } else if (!loader) {
    for (int i = threadIdx.x; i < S::Q_BYTES / 16; i += S::NW * 32)
      reinterpret_cast<uint4*>(sbase + S::Q_OFF)[i] = make_uint4(0, 0, 0, 0);
  }
  __syncthreads();
  if (warp < HG) {
    // head `warp`: its integer form in B rows warp (hi) and HG + warp (lo)
    constexpr int EPL = D / 32;  // elements per lane
    const __nv_bfloat16* qh = p.q + ((size_t)b * p.Hq + head0 + warp) * D + lane * EPL;
    float x[EPL];
    float amax = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      x[e] = __bfloat162float(qh[e]);
      amax = fmaxf(amax, fabsf(x[e]));
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    // amax < 2^E with E = biased exponent - 126; q * 2^(14 - E) lies in (-2^14, 2^14)
    int k = 14 - ((int)((__float_as_uint(amax) >> 23) & 0xFFu) - 126);
    k = max(-126, min(126, k));
    const float sq = __uint_as_float((uint32_t)(k + 127) << 23);
    if (lane == 0) cq[warp] = p.scale_log2 * __uint_as_float((uint32_t)(127 - k) << 23);
    uint32_t hi = 0, lo = 0;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      const int qi = __float2int_rn(x[e] * sq);
      const int h8 = (qi + 128) >> 8;
      const int l8 = qi - (h8 << 8);
      hi |= (uint32_t)(h8 & 0xFF) << (8 * e);
      lo |= (uint32_t)(l8 & 0xFF) << (8 * e);
    }
    unsigned char* qs = sbase + S::Q_OFF;
    const int d0 = lane * EPL;
    if constexpr (EPL == 4) {
      *reinterpret_cast<uint32_t*>(qs + swizzled_offset<D>(warp, d0)) = hi;
      *reinterpret_cast<uint32_t*>(qs + swizzled_offset<D>(HG + warp, d0)) = lo;
    } else {
      *reinterpret_cast<uint16_t*>(qs + swizzled_offset<D>(warp, d0)) = (uint16_t)hi;
      *reinterpret_cast<uint16_t*>(qs + swizzled_offset<D>(HG + warp, d0)) = (uint16_t)lo;
    }
  }
  if (!loader) fence_proxy_async_smem();  // the MMA reads the q rows (and zeros) through the async proxy
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  const int rows_cta = min(L - pg0 * kPageRows, n * kPageRows);
  const int lo_cta = WIN ? window_first_key(L, p.window) - pg0 * kPageRows : 0;
  LaneState<HG> st;
  st.reset();
  const int rg = lane / (D / 16), sub = lane % (D / 16);

  if (loader) {
    // ------------------------------------------------- loads and MMAs --
    int chunk = 0;
    auto validate = [&](int e, int c) {  // entries of the CTA's pages must lie in the pool
      if (c * 32 + lane < n && (e < 0 || e >= p.NB)) {
        set_error(PKV_ERR_BOUNDS);
        e = 0;
      }
      return e;
    };
    ent_cur = validate(ent_cur, 0);
    const uint64_t pol = policy_evict_first();
    auto issue = [&](int i) {  // warp-wide: tile i into stage i % ST
      const int c = i >> 2;    // 4 tiles per chunk of 32 entries
      if (c != chunk) {
        chunk = c;
        ent_cur = validate(ent_nxt, c);
        ent_nxt = load_raw(c + 1);
      }
      const int s = i % S::ST;
      const int np = min(S::TILE_PAGES, n - i * S::TILE_PAGES);
      // Copies are issued from two warps (K from one, V and the row scales
      // from the other): one thread's copies go out one after another, and
      // the tile's 16 page copies from one warp held the kernel back.
      const int blk = __shfl_sync(0xffffffffu, ent_cur, ((i & 3) << 3) + (lane & 7));
      if (lane == 0) mbar_arrive_expect_tx(full(s), np * S::PAGE);
      __syncwarp();
      if (lid == 0) {
        if (lane < np)
          tc::tma_load_4d(base + S::K_OFF + s * S::K_TILE + lane * S::PAGE, &tm_k, 0, 0, kvh, blk, full(s));
        return;
      }
      if (lane < np)
        bulk_g2s_hint(base + S::V_OFF + s * S::K_TILE + lane * S::PAGE,
                      p.v_cache + ((size_t)blk * p.Hkv + kvh) * S::PAGE, S::PAGE, full(s), pol);
      // Row scales, 64 bytes per page and pool: as bulk copies they would
      // double the copies of a tile, and a copy costs about the same whatever
      // its size, so the 32 lanes gather them 16 bytes each instead.
      const int pg = lane >> 2;  // page of this lane's two 16-byte pieces
      const int blk_s = __shfl_sync(0xffffffffu, ent_cur, ((i & 3) << 3) + pg);
      if (pg < np) {
        const size_t so = ((size_t)blk_s * p.Hkv + kvh) * kPageRows + (lane & 3) * 4;
        const uint32_t sc = base + S::S_OFF + s * S::SC_STAGE + lane * 16;
        cp_async16(sc, p.k_scale + so, pol);
        cp_async16(sc + S::TILE_ROWS * 4, p.v_scale + so, pol);
      }
      cp_async_arrive_noinc(full(s));
    };
    constexpr uint32_t IDESC = tc::idesc_s8_s32(S::TILE_ROWS, S::MMA_N);
    const uint64_t desc_k = tc::smem_desc_sw(base + S::K_OFF, 16, S::SBO, S::SW_LAYOUT);
    const uint64_t desc_q = tc::smem_desc_sw(base + S::Q_OFF, 16, S::SBO, S::SW_LAYOUT);
    int issued = 0, mmas = 0;
    auto mma = [&](int i) -> bool {  // scores of tile i into TMEM buffer i & 1
      bool good = true;
      if (lane == 0) {
        const int s = i % S::ST;
        good = mbar_wait(full(s), (i / S::ST) & 1);
        if (good && i >= 2) good = mbar_wait(sfree(i & 1), ((i - 2) >> 1) & 1);
        if (good) {
          tc::fence_after_sync();
          const uint32_t d = tmem + (i & 1) * S::MMA_N;
#pragma unroll
          for (int kk = 0; kk < S::KSTEPS; ++kk)
            tc::mma_i8_ss(d, desc_k + (uint64_t)((s * S::K_TILE + kk * 32) >> 4), desc_q + (uint64_t)(kk * 2),
                          IDESC, kk > 0 ? 1u : 0u);
          tc::commit(sfull(i & 1));
        }
      }
      return __shfl_sync(0xffffffffu, good ? 1 : 0, 0) != 0;
    };
    for (; issued < S::ST && issued < nt; ++issued) issue(issued);
    bool ok = true;
    if (lid == 0) {
      ok = mma(0);
      if (ok) mmas = 1;
    }
    // MMA i + 1 goes out while the consumers work on tile i; the stage of
    // tile i is refilled once they are done with it.
    for (int i = 0; ok && i < nt; ++i) {
      if (lid == 0 && i + 1 < nt) {
        ok = mma(i + 1);
        if (!ok) break;
        mmas = i + 2;
      }
      if (i + S::ST < nt) {
        bool good = true;
        if (lane == 0) good = mbar_wait(empty(i % S::ST), (i / S::ST) & 1);
        if (__shfl_sync(0xffffffffu, good ? 1 : 0, 0) == 0) {
          ok = false;
          break;
        }
        issue(i + S::ST);
        issued = i + S::ST + 1;
      }
    }
    if (!ok && lane == 0) {
      // after a timeout: let every issued copy land and every MMA finish
      // before the ring is reused and TMEM released
      for (int s = 0; s < S::ST && s < issued; ++s) {
        const int last = s + ((issued - 1 - s) / S::ST) * S::ST;
        mbar_wait(full(s), (last / S::ST) & 1);
      }
      if (mmas > 0) mbar_wait(sfull((mmas - 1) & 1), ((mmas - 1) >> 1) & 1);
    }
    __syncwarp();
  } else {
    // ----------------------------------------------------- consumers --
    float cqr[HG];
#pragma unroll
    for (int h = 0; h < HG; ++h) cqr[h] = cq[h];
    float* scw = reinterpret_cast<float*>(sbase + S::P_OFF) + warp * S::WROWS * 4;
    constexpr int RPW = 32 / (D / 16), TPL = S::WROWS / RPW;
    for (int i = 0; i < nt; ++i) {
      const int s = i % S::ST;
      if (!__all_sync(0xffffffffu, mbar_wait(sfull(i & 1), (i >> 1) & 1))) break;
      tc::fence_after_sync();
      uint32_t r[8];
      tc::ld_32x32b_x8(tmem + ((uint32_t)(32 * warp) << 16) + (i & 1) * S::MMA_N, r);
      tc::wait_ld();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(sfree(i & 1));
      // V codes and row scales of the tile (their copies completed before the MMA ran)
      if (!__all_sync(0xffffffffu, mbar_wait(full(s), (i / S::ST) & 1))) break;
      const int row0 = i * S::TILE_ROWS + warp * S::WROWS;  // CTA row of the warp's first key
      const int nvalid = rows_cta - row0, nstart = lo_cta - row0;
      const float* ksc = reinterpret_cast<const float*>(sbase + S::S_OFF + s * S::SC_STAGE) + warp * S::WROWS;
      {
        // This lane's key.  256 S_hi + S_lo is the exact integer q.k per head.
        // Its softmax weight is taken here once, not by each lane that
        // reads the row's V: the running max moves only when a score passes
        // it by more than 8 (log2), so weights stay below 2^8 and a move,
        // with its rescale, is rare after the first tile.
        const bool v = lane < nvalid && lane >= nstart;
        const float ks = v ? ksc[lane] : 0.f;  // rows outside the range are never read
        const float vs = v ? ksc[S::TILE_ROWS + lane] : 0.f;
        float sc[HG];
        bool big = false;
#pragma unroll
        for (int h = 0; h < HG; ++h) {
          sc[h] = v ? (float)((int)r[h] * 256 + (int)r[HG + h]) * (ks * cqr[h]) : -INFINITY;
          big |= sc[h] > st.m[h] + 8.f;
        }
        if (__any_sync(0xffffffffu, big)) {
#pragma unroll
          for (int h = 0; h < HG; ++h) {
            float mt = sc[h];
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
            const float mn = fmaxf(st.m[h], mt);
            const float alpha = (mn == -INFINITY) ? 1.f : ex2(st.m[h] - mn);
            st.m[h] = mn;
            st.l[h] *= alpha;
            const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
            for (int e = 0; e < 8; ++e) st.acc[h][e] = __fmul2_rn(st.acc[h][e], a2);
          }
        }
        float o[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          if (h < HG) {
            const float pr = v ? ex2(sc[h] - st.m[h]) : 0.f;
            st.l[h] += pr;      // this lane's keys only; summed over the warp at the end
            o[h] = pr * vs;     // the V scale rides on the weight
          } else {
            o[h] = 0.f;
          }
        }
        *reinterpret_cast<float4*>(scw + lane * 4) = make_float4(o[0], o[1], o[2], o[3]);
      }
      __syncwarp();
      // every row of the warp's slice: invalid rows carry weight 0 and their
      // codes are finite bytes, so no row needs a test
      const unsigned char* vp = sbase + S::V_OFF + s * S::K_TILE + warp * S::WROWS * D;
#pragma unroll
      for (int t = 0; t < TPL; ++t) {
        const int rr = rg + t * RPW;
        const float4 w4 = *reinterpret_cast<const float4*>(scw + rr * 4);
        const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
        const uint4 va = reinterpret_cast<const uint4*>(vp + rr * D)[sub];
        float2 v2[8];
        widen_i8x4(va.x, v2[0], v2[1]);
        widen_i8x4(va.y, v2[2], v2[3]);
        widen_i8x4(va.z, v2[4], v2[5]);
        widen_i8x4(va.w, v2[6], v2[7]);
#pragma unroll
        for (int h = 0; h < HG; ++h) {
          const float2 pp = make_float2(wv[h], wv[h]);
#pragma unroll
          for (int e = 0; e < 8; ++e) st.acc[h][e] = __ffma2_rn(pp, v2[e], st.acc[h][e]);
        }
      }
      // the stage is refilled by the copy engine after this: order the reads first
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(empty(s));
    }
  }

  // ---------------------------------------------------------- merge --
  launch_dependents();  // a merge launched after this kernel may be scheduled now
  tc::fence_before_sync();
  __syncthreads();  // every copy landed and every MMA finished (or was drained)
  if (loader) {
    if (lid == 0) {
      tc::fence_after_sync();
      tc::dealloc(tmem, S::TMEM_COLS);
    }
  } else {
    // the running max is the warp's; the sums are per key lane: total them,
    // held once per column of lanes so the row-group merge adds them once
#pragma unroll
    for (int h = 0; h < HG; ++h) {
      float l = st.l[h];
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
      st.l[h] = rg == 0 ? l : 0.f;
    }
    warp_merge<D, HG, false>(st);
    warp_store<D, HG>(reinterpret_cast<float*>(sbase + S::K_OFF) + warp * S::MERGE_STRIDE, st, rg, sub,
                      2 * sub, 2 * sub + 1);
  }
  __syncthreads();
  if (loader) return;
  const size_t row = (size_t)b * p.Hq + head0;
  const float* parts = reinterpret_cast<const float*>(sbase + S::K_OFF);
  if (p.num_splits == 1)
    cta_combine<D, HG, S::NW>(parts, S::MERGE_STRIDE, p.out + row * D, nullptr, 0, nullptr, 0);
  else
    cta_combine<D, HG, S::NW>(parts, S::MERGE_STRIDE, nullptr, p.o_part + (row * p.num_splits + split) * D,
                              (size_t)p.num_splits * D, p.lse_part + row * p.num_splits + split,
                              (size_t)p.num_splits);
}

}  // namespace pkv
