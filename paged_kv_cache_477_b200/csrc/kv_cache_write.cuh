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
