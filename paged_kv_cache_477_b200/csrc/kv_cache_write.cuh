// kv_cache_write.cuh -- scatter new K/V rows into physical cache slots.
//
// The paged cache maps a logical position to (physical block, offset) through
// a slot number slot = block * bs + offset ("从零构建CUDA推理引擎：Tiny-Infer
// 项目的技术深度解析", section "分页KV缓存：借鉴操作系统的内存管理").  This is
// a pure bit copy, so the result is exact.
//
// One thread moves one 16-byte vector (8 bf16) of K and the matching vector of
// V.  Consecutive threads walk a row, then the kv heads, then the tokens, so
// both the reads of key/value and the writes into a page are coalesced.  The
// work is tiny (a few hundred KB per decode step) and latency-bound: no shared
// memory staging would help it.
#pragma once
#include "pkv_common.cuh"

namespace pkv {

struct KvWriteParams {
  const uint4* key;        // [T][Hkv][D] bf16, viewed as 16-byte vectors
  const uint4* value;
  int64_t key_stride_vec;  // token stride in 16-byte vectors
  int64_t value_stride_vec;
  uint4* k_cache;          // [NB][Hkv][bs][D]
  uint4* v_cache;
  const int64_t* slot_mapping;
  int64_t total_vec;       // T * Hkv * D/8
  int64_t pool_slots;      // NB * bs
  int32_t Hkv, vec_per_row, bs;
};

__global__ void __launch_bounds__(256) kv_cache_write_kernel(const __grid_constant__ KvWriteParams p) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= p.total_vec) return;
  const int32_t c = (int32_t)(idx % p.vec_per_row);
  const int64_t th = idx / p.vec_per_row;
  const int32_t h = (int32_t)(th % p.Hkv);
  const int64_t t = th / p.Hkv;
  const int64_t slot = __ldg(p.slot_mapping + t);
  if (slot < 0) return;  // padding token
  if (slot >= p.pool_slots) {
    set_error(PKV_ERR_BOUNDS);
    return;
  }
  const int64_t blk = slot / p.bs, off = slot % p.bs;
  const int64_t dst = ((blk * p.Hkv + h) * p.bs + off) * p.vec_per_row + c;
  const uint4 kv = __ldg(p.key + t * p.key_stride_vec + (int64_t)h * p.vec_per_row + c);
  const uint4 vv = __ldg(p.value + t * p.value_stride_vec + (int64_t)h * p.vec_per_row + c);
  p.k_cache[dst] = kv;
  p.v_cache[dst] = vv;
}

}  // namespace pkv

namespace pkv {

// ---------------------------------------------------------------------------
// INT8 cache write: quantise each new (token, kv head) row of K and of V to
// int8 codes with one fp32 scale per row (Tiny-Infer page, section on INT8
// quantisation; the page fixes no granularity or rounding, so: symmetric,
// amax / 127, round half to even, all in fp32 -- the same operations, in the
// same order, as the reference definition, so codes and scales are exact).
//   amax = max |x|;  inv = 127 / amax;  code = clamp(rint(x * inv), +-127);
//   scale = amax / 127;  a zero row gives codes 0 and scale 0.
// One warp per row (K rows, then V rows); lane l holds elements
// [l * EPL, (l + 1) * EPL).  Non-finite inputs give unspecified codes.
// ---------------------------------------------------------------------------
struct KvWriteI8Params {
  const __nv_bfloat16* key;    // [T][Hkv][D], token stride given
  const __nv_bfloat16* value;
  int64_t key_stride, value_stride;  // elements
  int8_t* k_cache;             // [NB][Hkv][bs][D]
  int8_t* v_cache;
  float* k_scale;              // [NB][Hkv][bs]
  float* v_scale;
  const int64_t* slot_mapping;
  int64_t rows;                // 2 * T * Hkv
  int64_t pool_slots;          // NB * bs
  int32_t T, Hkv, D, bs;
};

template <int EPL>
__global__ void __launch_bounds__(256) kv_cache_write_i8_kernel(const __grid_constant__ KvWriteI8Params p) {
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= p.rows) return;
  const bool is_v = row >= (int64_t)p.T * p.Hkv;
  const int64_t th = is_v ? row - (int64_t)p.T * p.Hkv : row;
  const int32_t h = (int32_t)(th % p.Hkv);
  const int64_t t = th / p.Hkv;
  const int64_t slot = __ldg(p.slot_mapping + t);
  if (slot < 0) return;  // padding token
  if (slot >= p.pool_slots) {
    if (lane == 0) set_error(PKV_ERR_BOUNDS);
    return;
  }
  const __nv_bfloat16* src = (is_v ? p.value + t * p.value_stride : p.key + t * p.key_stride) +
                             (int64_t)h * p.D + lane * EPL;
  float x[EPL];
  float amax = 0.f;
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    x[e] = __bfloat162float(src[e]);
    amax = fmaxf(amax, fabsf(x[e]));
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const int64_t blk = slot / p.bs, off = slot % p.bs;
  const int64_t dst_row = (blk * p.Hkv + h) * p.bs + off;
  int8_t* dst = (is_v ? p.v_cache : p.k_cache) + dst_row * p.D + lane * EPL;
  const float inv = amax > 0.f ? __fdiv_rn(127.f, amax) : 0.f;
  int8_t c[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    const int r = __float2int_rn(__fmul_rn(x[e], inv));  // round half to even
    c[e] = (int8_t)max(-127, min(127, r));
  }
  if constexpr (EPL == 2) {
    *reinterpret_cast<uint16_t*>(dst) = (uint16_t)((uint8_t)c[0] | ((uint8_t)c[1] << 8));
  } else {
#pragma unroll
    for (int w = 0; w < EPL / 4; ++w)
      reinterpret_cast<uint32_t*>(dst)[w] = (uint32_t)(uint8_t)c[4 * w] | ((uint32_t)(uint8_t)c[4 * w + 1] << 8) |
                                            ((uint32_t)(uint8_t)c[4 * w + 2] << 16) |
                                            ((uint32_t)(uint8_t)c[4 * w + 3] << 24);
  }
  if (lane == 0) (is_v ? p.v_scale : p.k_scale)[dst_row] = amax > 0.f ? __fdiv_rn(amax, 127.f) : 0.f;
}

}  // namespace pkv

namespace pkv {

// ---------------------------------------------------------------------------
// Cache write with RoPE applied to K on the way in, so the rotated rows make
// one trip through memory (the fused-ops page fuses RoPE into the step before
// it, section 3.1).  The pages print no formula; Llama's form is used, as in
// the HuggingFace implementation the Tiny-Infer page checks against: element i
// < D/2 pairs with i + D/2 and turns by pos * base^(-2i/D):
//   k'[i] = k[i] cos - k[i + D/2] sin,   k'[i + D/2] = k[i + D/2] cos + k[i] sin.
// The angle is formed and reduced to [-pi, pi] in fp64 (an fp32 product of
// position and frequency would be off by ~1e-3 rad at 10^5 positions), then
// sine and cosine are taken in fp32 and the rotation is rounded once to bf16.
// V rows are copied.  One thread per (token, kv head, pair).
// ---------------------------------------------------------------------------
struct KvWriteRopeParams {
  const __nv_bfloat16* key;   // [T][Hkv][D], token stride given
  const __nv_bfloat16* value;
  int64_t key_stride, value_stride;  // elements
  __nv_bfloat16* k_cache;     // [NB][Hkv][bs][D]
  __nv_bfloat16* v_cache;
  const int64_t* slot_mapping;
  const int64_t* positions;   // [T]
  int64_t total;              // T * Hkv * D/2
  int64_t pool_slots;
  int32_t Hkv, D, bs;
  double log2_base;           // log2(rope base)
};

__global__ void __launch_bounds__(256) kv_cache_write_rope_kernel(const __grid_constant__ KvWriteRopeParams p) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= p.total) return;
  const int half = p.D / 2;
  const int i = (int)(idx % half);
  const int64_t th = idx / half;
  const int h = (int)(th % p.Hkv);
  const int64_t t = th / p.Hkv;
  const int64_t slot = __ldg(p.slot_mapping + t);
  if (slot < 0) return;  // padding token
  if (slot >= p.pool_slots) {
    if (i == 0) set_error(PKV_ERR_BOUNDS);
    return;
  }
  const int64_t pos = __ldg(p.positions + t);
  const double inv_freq = exp2(-2.0 * (double)i / (double)p.D * p.log2_base);
  const double a = (double)pos * inv_freq;
  const double two_pi = 6.283185307179586;
  const float r = (float)(a - two_pi * rint(a / two_pi));  // in [-pi, pi]
  float sn, cs;
  sincosf(r, &sn, &cs);
  const __nv_bfloat16* kr = p.key + t * p.key_stride + (int64_t)h * p.D;
  const __nv_bfloat16* vr = p.value + t * p.value_stride + (int64_t)h * p.D;
  const float x1 = __bfloat162float(kr[i]), x2 = __bfloat162float(kr[i + half]);
  const int64_t dst = ((slot / p.bs * p.Hkv + h) * p.bs + slot % p.bs) * p.D;
  p.k_cache[dst + i] = __float2bfloat16_rn(fmaf(x1, cs, -x2 * sn));
  p.k_cache[dst + i + half] = __float2bfloat16_rn(fmaf(x2, cs, x1 * sn));
  p.v_cache[dst + i] = vr[i];
  p.v_cache[dst + i + half] = vr[i + half];
}

}  // namespace pkv

namespace pkv {

// ---------------------------------------------------------------------------
// copy_blocks: for each (src, dst) pair copy a whole physical block (every kv
// head's page) of each of two pools, bit for bit -- the device half of
// copy-on-write for blocks shared between sequences (Tiny-Infer page,
// section "分页KV缓存：借鉴操作系统的内存管理").  One CTA per pair and pool,
// 16-byte vectors, coalesced.
// ---------------------------------------------------------------------------
struct CopyBlocksParams {
  uint4* pool[2];            // k and v (or codes and scales): [NB][block_vec] 16-byte vectors
  int64_t block_vec;         // 16-byte vectors per block
  const int32_t* pairs;      // [n][2]: src, dst
  int32_t n, NB;
};

__global__ void __launch_bounds__(256) copy_blocks_kernel(const __grid_constant__ CopyBlocksParams p) {
  const int pair = blockIdx.x, which = blockIdx.y;
  const int32_t src = __ldg(p.pairs + 2 * pair), dst = __ldg(p.pairs + 2 * pair + 1);
  if (src < 0 || src >= p.NB || dst < 0 || dst >= p.NB) {
    if (threadIdx.x == 0) set_error(PKV_ERR_BOUNDS);
    return;
  }
  const uint4* s = p.pool[which] + (int64_t)src * p.block_vec;
  uint4* d = p.pool[which] + (int64_t)dst * p.block_vec;
  for (int64_t i = threadIdx.x; i < p.block_vec; i += blockDim.x) d[i] = s[i];
}

}  // namespace pkv
