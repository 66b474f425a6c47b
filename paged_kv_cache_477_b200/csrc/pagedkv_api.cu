// pagedkv_api.cu -- the extern "C" boundary of libpagedkv.so.
//
// Host side only: validate arguments, pick a launch shape from host-known
// sizes (never from device data), enqueue kernels on the caller's stream.
// See include/pagedkv.h for the contract of every entry point.
#include <cuda_runtime.h>

#include <algorithm>
#include <new>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda.h>

#include "block_allocator.hpp"
#include "decode_attn.cuh"
#include "decode_attn_i8.cuh"
#include "lse_merge.cuh"
#include "hbm_probe.cuh"
#include "kv_cache_write.cuh"
#include "pkv_common.cuh"
#include "prefill_attn.cuh"

namespace {

thread_local int32_t t_launches = 0;

constexpr int kMaxDevices = 64;

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

pkv_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return dev;
}

int device_sm_count(int dev) {
  static int cache[kMaxDevices] = {0};
  if (dev < 0 || dev >= kMaxDevices) return 148;
  if (cache[dev] == 0) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
      sms = 148;
    cache[dev] = sms;
  }
  return cache[dev];
}

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

// ------------------------------------------------------------ tensor maps --
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// Tiled tensor map; dims/box innermost first, strides in bytes for dims
// 1..rank-1.  bf16 with a 128-byte swizzle unless told otherwise.
bool make_tmap(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims,
               const cuuint64_t* strides, const cuuint32_t* box,
               CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
               CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return false;
  const cuuint32_t elem_strides[5] = {1, 1, 1, 1, 1};
  return enc(map, dtype, (cuuint32_t)rank, const_cast<void*>(base), dims, strides, box, elem_strides,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


// ----------------------------------------------------------------- decode --
constexpr int kDecodeWarps = 4;
// Pages per ring stage and stages per warp, from B200 sweeps of the three
// decode workloads: D=128 one 8 KB page pair per stage, three stages; D=64
// three page pairs (48 key rows, 12 KB) per stage, two stages.  Either way
// 96 KB of pages are in flight per CTA, two CTAs per SM.  (D=64 with one page
// pair and six stages: 8 % slower; two pairs and three stages: 3 % slower.)
#ifndef PKV_DECODE_PPS64
#define PKV_DECODE_PPS64 3
#endif
#ifndef PKV_DECODE_STAGES64
#define PKV_DECODE_STAGES64 2
#endif
constexpr int pages_per_stage(int D) { return D == 128 ? 1 : PKV_DECODE_PPS64; }
constexpr int decode_stages(int D) { return D == 128 ? 3 : PKV_DECODE_STAGES64; }
// Copies are issued by producer warps, one per consumer warp (at D=64, twice
// the copies per byte: 3.78 -> 4.08 TB/s; at D=128 0.6-1.6 % faster).
constexpr bool decode_producers(int) { return true; }

template <int D, int HG>
using DecodeS = pkv::DecodeShape<D, HG, kDecodeWarps, decode_stages(D), pages_per_stage(D), decode_producers(D)>;

template <int D, int HG, bool WIN = false>
struct DecodeKernel {
  static constexpr auto fn =
      pkv::decode_attn_kernel<D, HG, kDecodeWarps, decode_stages(D), pages_per_stage(D), WIN, decode_producers(D)>;
  // set the dynamic shared-memory limit once per device; return CTAs per SM
  static int prepare(int dev) {
    static int occ[kMaxDevices] = {0};
    static std::mutex mu;
    if (dev < 0 || dev >= kMaxDevices) return 1;
    std::lock_guard<std::mutex> g(mu);
    if (occ[dev] == 0) {
      if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, DecodeS<D, HG>::SMEM_BYTES) !=
              cudaSuccess ||
          cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared) != cudaSuccess)
        return -1;
      if (decode_producers(D)) {
        // the producer form's setmaxnreg split is sized for exactly this
        // register count at launch; any other would leave it waiting forever
        cudaFuncAttributes attr;
        if (cudaFuncGetAttributes(&attr, fn) != cudaSuccess || attr.numRegs != DecodeS<D, HG>::REGS_LAUNCH)
          return -2;
      }
      int n = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, DecodeS<D, HG>::THREADS,
                                                        DecodeS<D, HG>::SMEM_BYTES) != cudaSuccess ||
          n <= 0)
        return -1;
      occ[dev] = n;
    }
    return occ[dev];
  }
};

int heads_per_cta(int G) {
  if (G % 4 == 0) return 4;
  if (G % 2 == 0) return 2;
  return 1;
}

int decode_occupancy(int D, int HG, int dev) {
  if (D == 128) {
    if (HG == 4) return DecodeKernel<128, 4>::prepare(dev);
    if (HG == 2) return DecodeKernel<128, 2>::prepare(dev);
    return DecodeKernel<128, 1>::prepare(dev);
  }
  if (HG == 4) return DecodeKernel<64, 4>::prepare(dev);
  if (HG == 2) return DecodeKernel<64, 2>::prepare(dev);
  return DecodeKernel<64, 1>::prepare(dev);
}

struct DecodePlan {
  int num_splits;
  int pages_per_split;
  size_t workspace;
};

int max_pages_of(int32_t MB, int32_t bs, int32_t hint) {
  const int64_t cap = (int64_t)MB * bs;
  const int64_t ctx = (hint > 0) ? std::min<int64_t>(hint, cap) : cap;
  return (int)((ctx + pkv::kPageRows - 1) / pkv::kPageRows);
}

size_t split_ws_bytes(int32_t B, int32_t Hq, int32_t D, int32_t C) {
  const size_t rows = (size_t)B * Hq * C;
  return round256(rows * D * sizeof(float)) + round256(rows * sizeof(float));
}

// Host-only choice of the split size.  Every CTA pays a few microseconds to
// start its copy stream and to merge at the end, so splits are kept long; a
// CTA streams ~40 GB/s when its SM is shared, so 96 pages (0.4-0.8 MB) take
// 10-20 us.  When the head groups alone give about three waves of CTAs the
// block scheduler balances them without splitting, unless a context can be
// long enough to leave one CTA running alone at the end: splits of up to
// kSplitPagesMany pages then.  The host sees only max_context_len, not the
// lengths themselves, so the rule is written for the longest context.
#ifndef PKV_SPLIT_PAGES
#define PKV_SPLIT_PAGES 96
#endif
#ifndef PKV_SPLIT_PAGES_MANY
#define PKV_SPLIT_PAGES_MANY 256
#endif
constexpr int kSplitPages = PKV_SPLIT_PAGES;
constexpr int kSplitPagesMany = PKV_SPLIT_PAGES_MANY;
// The int8 cache moves half the bytes per page, so its splits are longer
// (ragged long-context batch: 192 pages 94.6 us, 96 pages 102.7 us, 256 pages
// 96.7 us; the Llama-3.2-1B shape is the same at every size).
#ifndef PKV_SPLIT_PAGES_INT8
#define PKV_SPLIT_PAGES_INT8 192
#endif
constexpr int kWavesNoSplit = 3;

DecodePlan plan_auto(int32_t B, int32_t Hq, int32_t Hkv, int32_t D, int32_t MB, int32_t bs,
                     int32_t hint, bool int8 = false) {
  DecodePlan pl{1, std::max<int32_t>(MB, 1), 0};
  const int max_pages = max_pages_of(MB, bs, hint);
  const int G = Hq / Hkv, HG = heads_per_cta(G);
  const int64_t units = (int64_t)B * Hkv * (G / HG);
  const int dev = current_device();
  const int occ = std::max(1, decode_occupancy(D, HG, dev));
  const int64_t slots = (int64_t)device_sm_count(dev) * occ;
  if (units <= 0) return pl;
  const int target = units >= kWavesNoSplit * slots ? kSplitPagesMany : (int8 ? PKV_SPLIT_PAGES_INT8 : kSplitPages);
  const int C = (max_pages + target - 1) / target;
  if (C <= 1) return pl;
  const int pps = (max_pages + C - 1) / C;  // equal splits no longer than the target
  pl.pages_per_split = pps;
  pl.num_splits = (max_pages + pps - 1) / pps;
  pl.workspace = split_ws_bytes(B, Hq, D, pl.num_splits);
  return pl;
}

template <int D, int HG, bool WIN = false>
pkv_status launch_decode_t(const pkv::DecodeParams& p, int B, int Hkv, int nsub, int C, cudaStream_t st) {
  using K = DecodeKernel<D, HG, WIN>;
  const int occ = K::prepare(current_device());
  if (occ == -2) return PKV_ERR_UNSUPPORTED;  // a build whose register count the split does not fit
  if (occ < 0) return PKV_ERR_CUDA;
  dim3 grid(C, Hkv * nsub, B);
  K::fn<<<grid, DecodeS<D, HG>::THREADS, DecodeS<D, HG>::SMEM_BYTES, st>>>(p);
  return launch_status();
}

template <bool WIN>
pkv_status launch_decode_any(const pkv::DecodeParams& p, int D, int HG, int B, int Hkv, int nsub, int C,
                             cudaStream_t st) {
  if (D == 128)
    return HG == 4 ? launch_decode_t<128, 4, WIN>(p, B, Hkv, nsub, C, st)
           : HG == 2 ? launch_decode_t<128, 2, WIN>(p, B, Hkv, nsub, C, st)
                     : launch_decode_t<128, 1, WIN>(p, B, Hkv, nsub, C, st);
  return HG == 4 ? launch_decode_t<64, 4, WIN>(p, B, Hkv, nsub, C, st)
         : HG == 2 ? launch_decode_t<64, 2, WIN>(p, B, Hkv, nsub, C, st)
                   : launch_decode_t<64, 1, WIN>(p, B, Hkv, nsub, C, st);
}

// INT8 cache: Q.K^T on the tensor cores (decode_attn_i8.cuh)
template <int D, int HG, bool WIN>
struct DecodeI8Kernel {
  using S = pkv::DecodeI8Shape<D, HG>;
  static constexpr auto fn = pkv::decode_attn_i8_kernel<D, HG, WIN>;
  static bool prepare(int dev) {
    static int done[kMaxDevices] = {0};
    static std::mutex mu;
    if (dev < 0 || dev >= kMaxDevices) return false;
    std::lock_guard<std::mutex> g(mu);
    if (!done[dev]) {
      if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared) != cudaSuccess)
        return false;
      done[dev] = 1;
    }
    return true;
  }
};

template <int D, int HG, bool WIN>
pkv_status launch_decode_i8_t(const pkv::DecodeParams& p, int B, int Hkv, int nsub, int C, cudaStream_t st) {
  using K = DecodeI8Kernel<D, HG, WIN>;
  if (!K::prepare(current_device())) return PKV_ERR_CUDA;
  // K codes [NB][Hkv][16][D] bytes: one box is one page of one kv head.  With
  // no page to name (MB = 0) every context is empty and no copy is issued.
  CUtensorMap tm;
  std::memset(&tm, 0, sizeof tm);
  if (p.MB > 0) {
    const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)pkv::kPageRows, (cuuint64_t)Hkv, (cuuint64_t)p.NB};
    const cuuint64_t strides[3] = {(cuuint64_t)D, (cuuint64_t)pkv::kPageRows * D,
                                   (cuuint64_t)Hkv * pkv::kPageRows * D};
    const cuuint32_t box[4] = {(cuuint32_t)D, (cuuint32_t)pkv::kPageRows, 1, 1};
    if (!make_tmap(&tm, p.k_cache, 4, dims, strides, box, CU_TENSOR_MAP_DATA_TYPE_UINT8,
                   D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B))
      return PKV_ERR_CUDA;
  }
  dim3 grid(C, Hkv * nsub, B);
  K::fn<<<grid, K::S::THREADS, K::S::SMEM_BYTES, st>>>(p, tm);
  return launch_status();
}

template <bool WIN>
pkv_status launch_decode_i8(const pkv::DecodeParams& p, int D, int HG, int B, int Hkv, int nsub, int C,
                            cudaStream_t st) {
  if (D == 128)
    return HG == 4 ? launch_decode_i8_t<128, 4, WIN>(p, B, Hkv, nsub, C, st)
           : HG == 2 ? launch_decode_i8_t<128, 2, WIN>(p, B, Hkv, nsub, C, st)
                     : launch_decode_i8_t<128, 1, WIN>(p, B, Hkv, nsub, C, st);
  return HG == 4 ? launch_decode_i8_t<64, 4, WIN>(p, B, Hkv, nsub, C, st)
         : HG == 2 ? launch_decode_i8_t<64, 2, WIN>(p, B, Hkv, nsub, C, st)
                   : launch_decode_i8_t<64, 1, WIN>(p, B, Hkv, nsub, C, st);
}

// The merge is launched as a programmatic dependent of the split kernel: its
// grid is scheduled while the last split CTAs finish, and each merge CTA
// waits (griddepcontrol.wait) until the split kernel has completed and its
// partials are visible, so the launch gap between the two is hidden.
template <int D>
pkv_status launch_merge_t(const pkv::MergeParams& mp, int B, int Hq, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(Hq, B);
  cfg.blockDim = dim3(D);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, pkv::lse_merge_kernel<D>, mp) != cudaSuccess) return PKV_ERR_CUDA;
  return launch_status();
}

pkv_status check_decode_args(void* out, const void* q, const void* k_cache, const void* v_cache,
                             const int32_t* block_tables, int32_t MB, const int32_t* context_lens,
                             int32_t B, int32_t Hq, int32_t Hkv, int32_t D, int32_t NB, int32_t bs,
                             pkv_dtype dtype) {
  if (dtype != PKV_BF16) return PKV_ERR_UNSUPPORTED;
  if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || NB < 0 || MB < 0 || bs <= 0) return PKV_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return PKV_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return PKV_ERR_UNSUPPORTED;
  if (bs != pkv::kPageRows) return PKV_ERR_UNSUPPORTED;
  if (B == 0) return PKV_OK;
  if (!out || !q || !context_lens || ((MB > 0) && (!block_tables || !k_cache || !v_cache)))
    return PKV_ERR_INVALID_ARG;
  if (MB > 0 && NB == 0) return PKV_ERR_INVALID_ARG;  // no block a table entry could name
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
    return PKV_ERR_INVALID_ARG;
  return PKV_OK;
}

// k_scale / v_scale non-null: the int8 cache (codes in k_cache / v_cache).
pkv_status run_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                      const int32_t* block_tables, int32_t MB, const int32_t* context_lens,
                      int32_t B, int32_t Hq, int32_t Hkv, int32_t D, int32_t NB, float scale,
                      const DecodePlan& pl, void* workspace, cudaStream_t st,
                      const float* k_scale = nullptr, const float* v_scale = nullptr, int32_t window = 0) {
  const int G = Hq / Hkv, HG = heads_per_cta(G), nsub = G / HG;
  const int C = pl.num_splits;
  pkv::DecodeParams p{};
  p.out = static_cast<__nv_bfloat16*>(out);
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k_cache = static_cast<const unsigned char*>(k_cache);
  p.v_cache = static_cast<const unsigned char*>(v_cache);
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.NB = NB; p.MB = MB;
  p.G = G; p.nsub = nsub;
  p.pages_per_split = pl.pages_per_split;
  p.num_splits = C;
  p.cap_tokens = (int32_t)std::min<int64_t>((int64_t)MB, (int64_t)C * pl.pages_per_split) * pkv::kPageRows;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.window = window;
  // a window bounds the pages read, not the context: any length the table holds
  if (window > 0) p.cap_tokens = MB * pkv::kPageRows;
  if (C > 1) {
    const size_t rows = (size_t)B * Hq * C;
    p.o_part = static_cast<float*>(workspace);
    p.lse_part = reinterpret_cast<float*>(static_cast<unsigned char*>(workspace) +
                                          round256(rows * D * sizeof(float)));
  }
  pkv_status s = k_scale    ? (window > 0 ? launch_decode_i8<true>(p, D, HG, B, Hkv, nsub, C, st)
                                           : launch_decode_i8<false>(p, D, HG, B, Hkv, nsub, C, st))
                 : window > 0 ? launch_decode_any<true>(p, D, HG, B, Hkv, nsub, C, st)
                              : launch_decode_any<false>(p, D, HG, B, Hkv, nsub, C, st);
  if (s != PKV_OK) return s;
  int launches = 1;
  if (C > 1) {
    pkv::MergeParams mp{};
    mp.out = p.out;
    mp.o_part = p.o_part;
    mp.lse_part = p.lse_part;
    mp.context_lens = context_lens;
    mp.Hq = Hq;
    mp.num_splits = C;
    mp.pages_per_split = pl.pages_per_split;
    mp.cap_tokens = p.cap_tokens;
    mp.window = window;
    s = D == 128 ? launch_merge_t<128>(mp, B, Hq, st) : launch_merge_t<64>(mp, B, Hq, st);
    if (s != PKV_OK) return s;
    ++launches;
  }
  t_launches = launches;
  return PKV_OK;
}

// ---------------------------------------------------------------- prefill --
template <int D>
int prefill_prepare(int dev) {
  static int done[kMaxDevices] = {0};
  static std::mutex mu;
  if (dev < 0 || dev >= kMaxDevices) return -1;
  std::lock_guard<std::mutex> g(mu);
  if (!done[dev]) {
    for (const void* fn : {reinterpret_cast<const void*>(pkv::prefill_attn_kernel<D, false>),
                           reinterpret_cast<const void*>(pkv::prefill_attn_kernel<D, true>)}) {
      if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, pkv::pf::Layout<D>::SMEM_BYTES) !=
          cudaSuccess)
        return -1;
      // the kernel's setmaxnreg split is sized for exactly this register count
      cudaFuncAttributes attr;
      if (cudaFuncGetAttributes(&attr, fn) != cudaSuccess || attr.numRegs != pkv::pf::REGS_LAUNCH) return -2;
    }
    done[dev] = 1;
  }
  return 0;
}

__global__ void wait_timeout_selftest_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    pkv::mbar_init(pkv::smem_addr(&bar), 1);
    pkv::fence_barrier_init();
  }
  __syncthreads();
  // Nothing ever arrives on this barrier: the bounded wait must give up,
  // record PKV_ERR_TIMEOUT and return.
  if (threadIdx.x == 0) pkv::mbar_wait(pkv::smem_addr(&bar), 0, limit_ns);
}

}  // namespace

extern "C" {

const char* pkv_status_string(pkv_status s) {
  switch (s) {
    case PKV_OK: return "ok";
    case PKV_ERR_INVALID_ARG: return "invalid argument";
    case PKV_ERR_UNSUPPORTED: return "unsupported configuration";
    case PKV_ERR_CUDA: return "CUDA error";
    case PKV_ERR_TIMEOUT: return "device wait timed out";
    case PKV_ERR_BOUNDS: return "index out of range on the device";
    case PKV_ERR_WORKSPACE: return "workspace missing or too small";
    case PKV_ERR_NO_BLOCKS: return "not enough free blocks";
  }
  return "unknown status";
}

int32_t pkv_last_launch_count(void) { return t_launches; }

pkv_status pkv_kv_cache_write(const void* key, const void* value, int64_t key_stride_tok,
                              int64_t value_stride_tok, void* k_cache, void* v_cache,
                              const int64_t* slot_mapping, int32_t T, int32_t Hkv, int32_t D,
                              int32_t NB, int32_t bs, pkv_dtype dtype, pkv_stream_t stream) {
  t_launches = 0;
  if (dtype != PKV_BF16) return PKV_ERR_UNSUPPORTED;
  if (T < 0 || Hkv <= 0 || D <= 0 || NB < 0 || bs <= 0) return PKV_ERR_INVALID_ARG;
  if (D % 8 != 0) return PKV_ERR_UNSUPPORTED;
  if (T == 0) return PKV_OK;
  if (!key || !value || !k_cache || !v_cache || !slot_mapping) return PKV_ERR_INVALID_ARG;
  if (!aligned16(key) || !aligned16(value) || !aligned16(k_cache) || !aligned16(v_cache))
    return PKV_ERR_INVALID_ARG;
  if (key_stride_tok < (int64_t)Hkv * D || value_stride_tok < (int64_t)Hkv * D ||
      key_stride_tok % 8 != 0 || value_stride_tok % 8 != 0)
    return PKV_ERR_INVALID_ARG;
  pkv::KvWriteParams p{};
  p.key = static_cast<const uint4*>(key);
  p.value = static_cast<const uint4*>(value);
  p.key_stride_vec = key_stride_tok / 8;
  p.value_stride_vec = value_stride_tok / 8;
  p.k_cache = static_cast<uint4*>(k_cache);
  p.v_cache = static_cast<uint4*>(v_cache);
  p.slot_mapping = slot_mapping;
  p.vec_per_row = D / 8;
  p.total_vec = (int64_t)T * Hkv * p.vec_per_row;
  p.pool_slots = (int64_t)NB * bs;
  p.Hkv = Hkv;
  p.bs = bs;
  const int threads = 256;
  const int64_t blocks = (p.total_vec + threads - 1) / threads;
  if (blocks > INT32_MAX) return PKV_ERR_INVALID_ARG;
  pkv::kv_cache_write_kernel<<<(unsigned)blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(p);
  pkv_status s = launch_status();
  if (s == PKV_OK) t_launches = 1;
  return s;
}

pkv_status pkv_kv_cache_write_int8(const void* key, const void* value, int64_t key_stride_tok,
                                   int64_t value_stride_tok, void* k_cache, void* v_cache, float* k_scale,
                                   float* v_scale, const int64_t* slot_mapping, int32_t T, int32_t Hkv,
                                   int32_t D, int32_t NB, int32_t bs, pkv_stream_t stream) {
  t_launches = 0;
  if (T < 0 || Hkv <= 0 || D <= 0 || NB < 0 || bs <= 0) return PKV_ERR_INVALID_ARG;
  if (D != 64 && D != 128 && D != 256) return PKV_ERR_UNSUPPORTED;
  if (T == 0) return PKV_OK;
  if (!key || !value || !k_cache || !v_cache || !k_scale || !v_scale || !slot_mapping)
    return PKV_ERR_INVALID_ARG;
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k_scale) || !aligned16(v_scale) ||
      (reinterpret_cast<uintptr_t>(key) & 1) || (reinterpret_cast<uintptr_t>(value) & 1))
    return PKV_ERR_INVALID_ARG;
  if (key_stride_tok < (int64_t)Hkv * D || value_stride_tok < (int64_t)Hkv * D) return PKV_ERR_INVALID_ARG;
  pkv::KvWriteI8Params p{};
  p.key = static_cast<const __nv_bfloat16*>(key);
  p.value = static_cast<const __nv_bfloat16*>(value);
  p.key_stride = key_stride_tok;
  p.value_stride = value_stride_tok;
  p.k_cache = static_cast<int8_t*>(k_cache);
  p.v_cache = static_cast<int8_t*>(v_cache);
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  p.slot_mapping = slot_mapping;
  p.rows = 2 * (int64_t)T * Hkv;
  p.pool_slots = (int64_t)NB * bs;
  p.T = T; p.Hkv = Hkv; p.D = D; p.bs = bs;
  const int64_t blocks = (p.rows + 7) / 8;  // one warp per row, 8 warps per block
  if (blocks > INT32_MAX) return PKV_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (D == 64)
    pkv::kv_cache_write_i8_kernel<2><<<(unsigned)blocks, 256, 0, st>>>(p);
  else if (D == 128)
    pkv::kv_cache_write_i8_kernel<4><<<(unsigned)blocks, 256, 0, st>>>(p);
  else
    pkv::kv_cache_write_i8_kernel<8><<<(unsigned)blocks, 256, 0, st>>>(p);
  pkv_status s = launch_status();
  if (s == PKV_OK) t_launches = 1;
  return s;
}

pkv_status pkv_paged_attention_int8(void* out, const void* q, const void* k_cache, const void* v_cache,
                                    const float* k_scale, const float* v_scale, const int32_t* block_tables,
                                    int32_t MB, const int32_t* context_lens, int32_t B, int32_t Hq,
                                    int32_t Hkv, int32_t D, int32_t NB, int32_t bs, float scale,
                                    int32_t max_context_len_hint, void* workspace, size_t workspace_bytes,
                                    pkv_stream_t stream) {
  t_launches = 0;
  pkv_status s = check_decode_args(out, q, k_cache, v_cache, block_tables, MB, context_lens, B, Hq,
                                    Hkv, D, NB, bs, PKV_BF16);
  if (s != PKV_OK || B == 0) return s;
  if (MB > 0 && (!k_scale || !v_scale || !aligned16(k_scale) || !aligned16(v_scale)))
    return PKV_ERR_INVALID_ARG;
  DecodePlan pl = plan_auto(B, Hq, Hkv, D, MB, bs, max_context_len_hint, true);
  if (pl.num_splits > 1 && (!workspace || workspace_bytes < pl.workspace || !aligned16(workspace)))
    pl = DecodePlan{1, std::max<int32_t>(MB, 1), 0};  // no room: one CTA per head group
  if (pl.num_splits == 1) pl.pages_per_split = std::max<int32_t>(MB, 1);
  // a never-read dummy keeps the kernel on its int8 path when MB = 0
  static const float kNoScale[4] = {0.f, 0.f, 0.f, 0.f};
  return run_decode(out, q, k_cache, v_cache, block_tables, MB, context_lens, B, Hq, Hkv, D, NB, scale, pl,
                    workspace, static_cast<cudaStream_t>(stream), k_scale ? k_scale : kNoScale,
                    v_scale ? v_scale : kNoScale);
}

// pages a window of W keys can touch: W keys starting anywhere in a page
int window_pages(int32_t window) { return (int)(((int64_t)window + pkv::kPageRows - 2) / pkv::kPageRows) + 1; }

pkv_status pkv_paged_attention_int8_window(void* out, const void* q, const void* k_cache, const void* v_cache,
                                           const float* k_scale, const float* v_scale,
                                           const int32_t* block_tables, int32_t MB, const int32_t* context_lens,
                                           int32_t B, int32_t Hq, int32_t Hkv, int32_t D, int32_t NB, int32_t bs,
                                           float scale, int32_t window, void* workspace, size_t workspace_bytes,
                                           pkv_stream_t stream) {
  t_launches = 0;
  pkv_status s = check_decode_args(out, q, k_cache, v_cache, block_tables, MB, context_lens, B, Hq,
                                    Hkv, D, NB, bs, PKV_BF16);
  if (s != PKV_OK || B == 0) return s;
  if (window < 1) return PKV_ERR_INVALID_ARG;
  if (MB > 0 && (!k_scale || !v_scale || !aligned16(k_scale) || !aligned16(v_scale)))
    return PKV_ERR_INVALID_ARG;
  // the plan of pkv_paged_attention_window (split sizes for this kernel):
  // over the pages a window touches
  const int32_t span = (int32_t)std::min<int64_t>((int64_t)window_pages(window) * bs, (int64_t)MB * bs);
  DecodePlan pl = plan_auto(B, Hq, Hkv, D, MB, bs, span, true);
  if (pl.num_splits > 1 && (!workspace || workspace_bytes < pl.workspace || !aligned16(workspace)))
    pl = DecodePlan{1, std::max<int32_t>(MB, 1), 0};  // no room: one CTA per head group
  if (pl.num_splits == 1) pl.pages_per_split = std::max<int32_t>(MB, 1);
  static const float kNoScale[4] = {0.f, 0.f, 0.f, 0.f};
  return run_decode(out, q, k_cache, v_cache, block_tables, MB, context_lens, B, Hq, Hkv, D, NB, scale, pl,
                    workspace, static_cast<cudaStream_t>(stream), k_scale ? k_scale : kNoScale,
                    v_scale ? v_scale : kNoScale, window);
}

pkv_status pkv_paged_attention_window(void* out, const void* q, const void* k_cache, const void* v_cache,
                                      const int32_t* block_tables, int32_t MB, const int32_t* context_lens,
                                      int32_t B, int32_t Hq, int32_t Hkv, int32_t D, int32_t NB, int32_t bs,
                                      float scale, int32_t window, void* workspace, size_t workspace_bytes,
                                      pkv_dtype dtype, pkv_stream_t stream) {
  t_launches = 0;
  pkv_status s = check_decode_args(out, q, k_cache, v_cache, block_tables, MB, context_lens, B, Hq,
                                    Hkv, D, NB, bs, dtype);
  if (s != PKV_OK || B == 0) return s;
  if (window < 1) return PKV_ERR_INVALID_ARG;
  // plan over the pages a window touches; the kernel starts each sequence at
  // the first page its window reaches
  const int32_t span = (int32_t)std::min<int64_t>((int64_t)window_pages(window) * bs, (int64_t)MB * bs);
  DecodePlan pl = plan_auto(B, Hq, Hkv, D, MB, bs, span);
  if (pl.num_splits > 1 && (!workspace || workspace_bytes < pl.workspace || !aligned16(workspace)))
    pl = DecodePlan{1, std::max<int32_t>(MB, 1), 0};  // no room: one CTA per head group
  if (pl.num_splits == 1) pl.pages_per_split = std::max<int32_t>(MB, 1);
  return run_decode(out, q, k_cache, v_cache, block_tables, MB, context_lens, B, Hq, Hkv, D, NB, scale, pl,
                    workspace, static_cast<cudaStream_t>(stream), nullptr, nullptr, window);
}

size_t pkv_paged_attention_window_workspace_size(int32_t B, int32_t Hq, int32_t Hkv, int32_t D, int32_t MB,
                                                 int32_t bs, int32_t window) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || (D != 64 && D != 128) || bs != pkv::kPageRows || window < 1)
    return 0;
  const int32_t span = (int32_t)std::min<int64_t>((int64_t)window_pages(window) * bs, (int64_t)MB * bs);
  // enough for the bf16 and the int8 kernel's plans alike
  return std::max(plan_auto(B, Hq, Hkv, D, MB, bs, span).workspace,
                  plan_auto(B, Hq, Hkv, D, MB, bs, span, true).workspace);
}

pkv_status pkv_kv_cache_write_rope(const void* key, const void* value, int64_t key_stride_tok,
                                   int64_t value_stride_tok, void* k_cache, void* v_cache,
                                   const int64_t* slot_mapping, const int64_t* positions, int32_t T,
                                   int32_t Hkv, int32_t D, int32_t NB, int32_t bs, double rope_base,
                                   pkv_dtype dtype, pkv_stream_t stream) {
  t_launches = 0;
  if (dtype != PKV_BF16) return PKV_ERR_UNSUPPORTED;
  if (T < 0 || Hkv <= 0 || D <= 0 || D % 2 != 0 || NB < 0 || bs <= 0 || !(rope_base > 1.0) ||
      !std::isfinite(rope_base))
    return PKV_ERR_INVALID_ARG;
  if (T == 0) return PKV_OK;
  if (!key || !value || !k_cache || !v_cache || !slot_mapping || !positions) return PKV_ERR_INVALID_ARG;
  if (((reinterpret_cast<uintptr_t>(key) | reinterpret_cast<uintptr_t>(value) |
        reinterpret_cast<uintptr_t>(k_cache) | reinterpret_cast<uintptr_t>(v_cache)) & 1) != 0)
    return PKV_ERR_INVALID_ARG;
  if (key_stride_tok < (int64_t)Hkv * D || value_stride_tok < (int64_t)Hkv * D) return PKV_ERR_INVALID_ARG;
  pkv::KvWriteRopeParams p{};
  p.key = static_cast<const __nv_bfloat16*>(key);
  p.value = static_cast<const __nv_bfloat16*>(value);
  p.key_stride = key_stride_tok;
  p.value_stride = value_stride_tok;
  p.k_cache = static_cast<__nv_bfloat16*>(k_cache);
  p.v_cache = static_cast<__nv_bfloat16*>(v_cache);
  p.slot_mapping = slot_mapping;
  p.positions = positions;
  p.total = (int64_t)T * Hkv * (D / 2);
  p.pool_slots = (int64_t)NB * bs;
  p.Hkv = Hkv; p.D = D; p.bs = bs;
  p.log2_base = std::log2(rope_base);
  const int64_t blocks = (p.total + 255) / 256;
  if (blocks > INT32_MAX) return PKV_ERR_INVALID_ARG;
  pkv::kv_cache_write_rope_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
  pkv_status s = launch_status();
  if (s == PKV_OK) t_launches = 1;
  return s;
}

// ------------------------------------------------------- shared blocks --
struct pkv_block_allocator {
  pkv::BlockAllocator impl;
  explicit pkv_block_allocator(int32_t n) : impl(n) {}
};

pkv_status pkv_block_allocator_create(int32_t num_blocks, pkv_block_allocator** out) {
  if (!out || num_blocks < 0) return PKV_ERR_INVALID_ARG;
  *out = new (std::nothrow) pkv_block_allocator(num_blocks);
  return *out ? PKV_OK : PKV_ERR_INVALID_ARG;
}

void pkv_block_allocator_destroy(pkv_block_allocator* a) { delete a; }

pkv_status pkv_block_allocator_alloc(pkv_block_allocator* a, int32_t n, int32_t* ids) {
  if (!a || n < 0 || (n > 0 && !ids)) return PKV_ERR_INVALID_ARG;
  return a->impl.alloc(n, ids) ? PKV_OK : PKV_ERR_NO_BLOCKS;
}

pkv_status pkv_block_allocator_share(pkv_block_allocator* a, const int32_t* ids, int32_t n) {
  if (!a || n < 0 || (n > 0 && !ids)) return PKV_ERR_INVALID_ARG;
  return a->impl.share(ids, n) ? PKV_OK : PKV_ERR_INVALID_ARG;
}

pkv_status pkv_block_allocator_release(pkv_block_allocator* a, const int32_t* ids, int32_t n) {
  if (!a || n < 0 || (n > 0 && !ids)) return PKV_ERR_INVALID_ARG;
  return a->impl.release(ids, n) ? PKV_OK : PKV_ERR_INVALID_ARG;
}

pkv_status pkv_block_allocator_cow(pkv_block_allocator* a, int32_t id, int32_t* new_id, int32_t* must_copy) {
  if (!a || !new_id || !must_copy) return PKV_ERR_INVALID_ARG;
  if (a->impl.refcount(id) <= 0) return PKV_ERR_INVALID_ARG;
  bool copy = false;
  int32_t nid = -1;
  if (!a->impl.copy_on_write(id, &nid, &copy)) return PKV_ERR_NO_BLOCKS;
  *new_id = nid;
  *must_copy = copy ? 1 : 0;
  return PKV_OK;
}

int32_t pkv_block_allocator_num_free(pkv_block_allocator* a) { return a ? a->impl.num_free() : -1; }

int32_t pkv_block_allocator_refcount(pkv_block_allocator* a, int32_t id) { return a ? a->impl.refcount(id) : -1; }

pkv_status pkv_hbm_read_probe(const void* buf, size_t bytes, int32_t chunk_bytes, uint32_t* sink, int32_t nsink,
                              pkv_stream_t stream) {
  t_launches = 0;
  if (!buf || !sink || nsink <= 0 || bytes == 0 || bytes % 16 != 0 || !aligned16(buf))
    return PKV_ERR_INVALID_ARG;
  if (chunk_bytes < 4096 || chunk_bytes > pkv::kProbeRing / 3 || pkv::kProbeRing % chunk_bytes != 0)
    return PKV_ERR_INVALID_ARG;
  {
    static int ready[kMaxDevices] = {0};
    static std::mutex mu;
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return PKV_ERR_CUDA;
    std::lock_guard<std::mutex> g(mu);
    if (!ready[dev]) {
      if (cudaFuncSetAttribute(pkv::hbm_read_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               pkv::kProbeSmem) != cudaSuccess)
        return PKV_ERR_CUDA;
      ready[dev] = 1;
    }
  }
  pkv::hbm_read_probe_kernel<<<nsink, 32, pkv::kProbeSmem, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const unsigned char*>(buf), (int64_t)bytes, chunk_bytes, sink);
  pkv_status s = launch_status();
  if (s == PKV_OK) t_launches = 1;
  return s;
}

pkv_status pkv_copy_blocks(void* k_cache, void* v_cache, size_t block_bytes, const int32_t* pairs, int32_t n,
                           int32_t NB, pkv_stream_t stream) {
  t_launches = 0;
  if (n < 0 || NB < 0 || block_bytes == 0 || block_bytes % 16 != 0) return PKV_ERR_INVALID_ARG;
  if (n == 0) return PKV_OK;
  if (!k_cache || !v_cache || !pairs || !aligned16(k_cache) || !aligned16(v_cache)) return PKV_ERR_INVALID_ARG;
  if (n > 65535 * 64) return PKV_ERR_UNSUPPORTED;
  pkv::CopyBlocksParams p{};
  p.pool[0] = static_cast<uint4*>(k_cache);
  p.pool[1] = static_cast<uint4*>(v_cache);
  p.block_vec = (int64_t)(block_bytes / 16);
  p.pairs = pairs;
  p.n = n;
  p.NB = NB;
  pkv::copy_blocks_kernel<<<dim3(n, 2), 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
  pkv_status s = launch_status();
  if (s == PKV_OK) t_launches = 1;
  return s;
}

size_t pkv_split_workspace_size(int32_t B, int32_t Hq, int32_t D, int32_t num_splits) {
  if (B <= 0 || Hq <= 0 || D <= 0 || num_splits <= 1) return 0;
  return split_ws_bytes(B, Hq, D, num_splits);
}

size_t pkv_paged_attention_workspace_size(int32_t B, int32_t Hq, int32_t Hkv, int32_t D,
                                          int32_t MB, int32_t bs, int32_t max_context_len_hint) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || (D != 64 && D != 128) || bs != pkv::kPageRows)
    return 0;
  // enough for the bf16 and the int8 kernel's plans alike
  return std::max(plan_auto(B, Hq, Hkv, D, MB, bs, max_context_len_hint).workspace,
                  plan_auto(B, Hq, Hkv, D, MB, bs, max_context_len_hint, true).workspace);
}

pkv_status pkv_paged_attention(void* out, const void* q, const void* k_cache, const void* v_cache,
                               const int32_t* block_tables, int32_t MB,
                               const int32_t* context_lens, int32_t B, int32_t Hq, int32_t Hkv,
                               int32_t D, int32_t NB, int32_t bs, float scale,
                               int32_t max_context_len_hint, void* workspace,
                               size_t workspace_bytes, pkv_dtype dtype, pkv_stream_t stream) {
  t_launches = 0;
  pkv_status s = check_decode_args(out, q, k_cache, v_cache, block_tables, MB, context_lens, B, Hq,
                                    Hkv, D, NB, bs, dtype);
  if (s != PKV_OK || B == 0) return s;
  DecodePlan pl = plan_auto(B, Hq, Hkv, D, MB, bs, max_context_len_hint);
  if (pl.num_splits > 1 && (!workspace || workspace_bytes < pl.workspace || !aligned16(workspace)))
    pl = DecodePlan{1, std::max<int32_t>(MB, 1), 0};  // no room: one CTA per head group
  if (pl.num_splits == 1) pl.pages_per_split = std::max<int32_t>(MB, 1);
  return run_decode(out, q, k_cache, v_cache, block_tables, MB, context_lens, B, Hq, Hkv, D, NB,
                    scale, pl, workspace, static_cast<cudaStream_t>(stream));
}

pkv_status pkv_paged_attention_split(void* out, const void* q, const void* k_cache,
                                     const void* v_cache, const int32_t* block_tables, int32_t MB,
                                     const int32_t* context_lens, int32_t B, int32_t Hq,
                                     int32_t Hkv, int32_t D, int32_t NB, int32_t bs, float scale,
                                     int32_t max_context_len_hint, int32_t pages_per_split,
                                     void* workspace, size_t workspace_bytes, pkv_dtype dtype,
                                     pkv_stream_t stream) {
  t_launches = 0;
  pkv_status s = check_decode_args(out, q, k_cache, v_cache, block_tables, MB, context_lens, B, Hq,
                                    Hkv, D, NB, bs, dtype);
  if (s != PKV_OK) return s;
  if (pages_per_split <= 0) return PKV_ERR_INVALID_ARG;
  if (B == 0) return PKV_OK;
  const int max_pages = std::max(1, max_pages_of(MB, bs, max_context_len_hint));
  DecodePlan pl{(max_pages + pages_per_split - 1) / pages_per_split, pages_per_split, 0};
  if (pl.num_splits > 1) {
    pl.workspace = split_ws_bytes(B, Hq, D, pl.num_splits);
    if (!workspace || workspace_bytes < pl.workspace || !aligned16(workspace))
      return PKV_ERR_WORKSPACE;
  }
  return run_decode(out, q, k_cache, v_cache, block_tables, MB, context_lens, B, Hq, Hkv, D, NB,
                    scale, pl, workspace, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {
pkv_status prefill_impl(void* out, const void* q, const int32_t* query_start_loc, const void* k_cache,
                        const void* v_cache, const int32_t* block_tables, int32_t MB,
                        const int32_t* context_lens, int32_t B, int32_t sumQ, int32_t max_q_len, int32_t Hq,
                        int32_t Hkv, int32_t D, int32_t NB, int32_t bs, float scale, int32_t window,
                        pkv_dtype dtype, pkv_stream_t stream) {
  t_launches = 0;
  if (dtype != PKV_BF16) return PKV_ERR_UNSUPPORTED;
  if (B < 0 || sumQ < 0 || max_q_len < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || NB < 0 || MB < 0 || bs <= 0)
    return PKV_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return PKV_ERR_INVALID_ARG;
  const int G = Hq / Hkv;
  if ((D != 64 && D != 128) || bs != pkv::kPageRows || G > pkv::pf::BM)
    return PKV_ERR_UNSUPPORTED;
  if (!std::isfinite(scale)) return PKV_ERR_INVALID_ARG;
  if (B == 0 || sumQ == 0 || max_q_len == 0) return PKV_OK;
  if (!out || !q || !query_start_loc || !k_cache || !v_cache || !block_tables || !context_lens ||
      NB == 0 || MB == 0)
    return PKV_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
    return PKV_ERR_INVALID_ARG;
  const int dev = current_device();
  const int prep = D == 128 ? prefill_prepare<128>(dev) : prefill_prepare<64>(dev);
  if (prep == -2) return PKV_ERR_UNSUPPORTED;  // build with an unexpected register count
  if (prep < 0) return PKV_ERR_CUDA;

  CUtensorMap tm_q, tm_k, tm_v;
  {
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hq, (cuuint64_t)sumQ};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hq * D * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)G, (cuuint32_t)(pkv::pf::BM / G)};
    if (!make_tmap(&tm_q, q, 3, dims, strides, box)) return PKV_ERR_CUDA;
  }
  {
    const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)bs, (cuuint64_t)Hkv, (cuuint64_t)NB};
    const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)bs * D * 2, (cuuint64_t)Hkv * bs * D * 2};
    const cuuint32_t box[4] = {64, (cuuint32_t)bs, 1, 1};
    if (!make_tmap(&tm_k, k_cache, 4, dims, strides, box)) return PKV_ERR_CUDA;
    if (!make_tmap(&tm_v, v_cache, 4, dims, strides, box)) return PKV_ERR_CUDA;
  }
  pkv::PrefillParams p{};
  p.out = static_cast<__nv_bfloat16*>(out);
  p.query_start_loc = query_start_loc;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.NB = NB; p.MB = MB; p.G = G; p.sumQ = sumQ;
  p.scale_log2 = scale * 1.4426950408889634f;
  const int ppc = pkv::pf::NQT * (pkv::pf::BM / G);  // query positions per CTA
  // Query-tile pairs are the fastest grid dimension, so the CTAs of one
  // (sequence, kv head) are scheduled together and share its K/V pages
  // through L2; within a group the last pair (most keys) goes first.
  const int nct = (max_q_len + ppc - 1) / ppc;
  if (Hkv > 65535 || B > 65535) return PKV_ERR_UNSUPPORTED;
  p.nct = nct;
  p.window = window;
  dim3 grid(nct, Hkv, B);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  constexpr int S128 = pkv::pf::Layout<128>::SMEM_BYTES, S64 = pkv::pf::Layout<64>::SMEM_BYTES;
  if (D == 128) {
    if (window > 0)
      pkv::prefill_attn_kernel<128, true><<<grid, pkv::pf::THREADS, S128, st>>>(p, tm_q, tm_k, tm_v);
    else
      pkv::prefill_attn_kernel<128, false><<<grid, pkv::pf::THREADS, S128, st>>>(p, tm_q, tm_k, tm_v);
  } else {
    if (window > 0)
      pkv::prefill_attn_kernel<64, true><<<grid, pkv::pf::THREADS, S64, st>>>(p, tm_q, tm_k, tm_v);
    else
      pkv::prefill_attn_kernel<64, false><<<grid, pkv::pf::THREADS, S64, st>>>(p, tm_q, tm_k, tm_v);
  }
  pkv_status s = launch_status();
  if (s == PKV_OK) t_launches = 1;
  return s;
}

}  // namespace

extern "C" {

pkv_status pkv_paged_attention_prefill(void* out, const void* q, const int32_t* query_start_loc,
                                       const void* k_cache, const void* v_cache,
                                       const int32_t* block_tables, int32_t MB,
                                       const int32_t* context_lens, int32_t B, int32_t sumQ,
                                       int32_t max_q_len, int32_t Hq, int32_t Hkv, int32_t D,
                                       int32_t NB, int32_t bs, float scale, pkv_dtype dtype,
                                       pkv_stream_t stream) {
  return prefill_impl(out, q, query_start_loc, k_cache, v_cache, block_tables, MB, context_lens, B, sumQ,
                      max_q_len, Hq, Hkv, D, NB, bs, scale, 0, dtype, stream);
}

pkv_status pkv_paged_attention_prefill_window(void* out, const void* q, const int32_t* query_start_loc,
                                              const void* k_cache, const void* v_cache,
                                              const int32_t* block_tables, int32_t MB,
                                              const int32_t* context_lens, int32_t B, int32_t sumQ,
                                              int32_t max_q_len, int32_t Hq, int32_t Hkv, int32_t D,
                                              int32_t NB, int32_t bs, float scale, int32_t window,
                                              pkv_dtype dtype, pkv_stream_t stream) {
  if (window < 1) {
    t_launches = 0;
    return PKV_ERR_INVALID_ARG;
  }
  return prefill_impl(out, q, query_start_loc, k_cache, v_cache, block_tables, MB, context_lens, B, sumQ,
                      max_q_len, Hq, Hkv, D, NB, bs, scale, window, dtype, stream);
}

pkv_status pkv_get_device_error(pkv_stream_t stream, int32_t* err_out) {
  if (!err_out) return PKV_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return PKV_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, pkv::g_error_word, sizeof(int)) != cudaSuccess) return PKV_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(pkv::g_error_word, &zero, sizeof(int)) != cudaSuccess) return PKV_ERR_CUDA;
  *err_out = v;
  return PKV_OK;
}

pkv_status pkv_selftest_wait_timeout(uint32_t timeout_us, pkv_stream_t stream) {
  t_launches = 0;
  if (timeout_us == 0 || timeout_us > 5000000u) return PKV_ERR_INVALID_ARG;
  wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      (uint64_t)timeout_us * 1000ull);
  pkv_status s = launch_status();
  if (s == PKV_OK) t_launches = 1;
  return s;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Split-KV decode without any allocation by the caller.
//
// Some callers cannot hand the library a workspace: engine plugins whose
// enqueue hook must not allocate, serving loops that cannot afford the device
// synchronisation a cudaMalloc may cause, or processes whose device memory is
// already reserved in full by another allocator.  For them the split-KV
// partials live in this file-scope device array instead.  It is created when
// the library's device code is loaded on a GPU and stays there until the
// process exits (PKV_NOALLOC_SCRATCH_BYTES on every GPU that loads it).
// ---------------------------------------------------------------------------
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[PKV_NOALLOC_SCRATCH_BYTES];

// Host code cannot use g_noalloc_scratch's name as a device address: on the
// host it only stands in for the symbol.  Its device address is looked up once
// per device, with that device current, and kept here.
void* noalloc_scratch_address(int dev) {
  static void* addr[kMaxDevices] = {nullptr};
  static std::mutex mu;
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> g(mu);
  if (addr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) return nullptr;
    addr[dev] = ptr;
  }
  return addr[dev];
}

}  // namespace

extern "C" pkv_status pkv_paged_attention_split_noalloc(
    void* out, const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
    int32_t MB, const int32_t* context_lens, int32_t B, int32_t Hq, int32_t Hkv, int32_t D, int32_t NB,
    int32_t bs, float scale, int32_t max_context_len_hint, int32_t pages_per_split, pkv_dtype dtype,
    pkv_stream_t stream) {
  t_launches = 0;
  pkv_status s = check_decode_args(out, q, k_cache, v_cache, block_tables, MB, context_lens, B, Hq,
                                    Hkv, D, NB, bs, dtype);
  if (s != PKV_OK) return s;
  if (pages_per_split <= 0) return PKV_ERR_INVALID_ARG;
  if (B == 0) return PKV_OK;
  const int max_pages = std::max(1, max_pages_of(MB, bs, max_context_len_hint));
  DecodePlan pl{(max_pages + pages_per_split - 1) / pages_per_split, pages_per_split, 0};
  void* scratch = nullptr;
  if (pl.num_splits > 1) {
    pl.workspace = split_ws_bytes(B, Hq, D, pl.num_splits);
    if (pl.workspace > (size_t)PKV_NOALLOC_SCRATCH_BYTES) return PKV_ERR_WORKSPACE;
    scratch = noalloc_scratch_address(current_device());
    if (scratch == nullptr) return PKV_ERR_CUDA;
  }
  return run_decode(out, q, k_cache, v_cache, block_tables, MB, context_lens, B, Hq, Hkv, D, NB,
                    scale, pl, scratch, static_cast<cudaStream_t>(stream));
}
