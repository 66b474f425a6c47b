// block_allocator.hpp -- host-side allocator of physical cache blocks with
// reference counts, for blocks shared between sequences.
//
// The paged cache maps each sequence's logical pages to physical blocks
// through its block table; sequences that share a prefix (parallel sampling
// from one prompt) can point at the same physical blocks and copy a block
// only when one of them is about to write into it ("从零构建CUDA推理引擎：
// Tiny-Infer项目的技术深度解析", section "分页KV缓存：借鉴操作系统的内存管理",
// which plans vLLM-style block copying for parallel sampling).
//
// Host only; no CUDA.  A free list (stack, lowest ids handed out first on a
// fresh allocator) and a reference count per block; every call is guarded by
// one mutex, so one allocator may serve several host threads.
#pragma once
#include <cstdint>
#include <mutex>
#include <vector>

namespace pkv {

class BlockAllocator {
 public:
  explicit BlockAllocator(int32_t num_blocks) : refs_(num_blocks, 0) {
    free_.reserve(num_blocks);
    for (int32_t b = num_blocks - 1; b >= 0; --b) free_.push_back(b);
  }

  int32_t num_blocks() const { return (int32_t)refs_.size(); }

  int32_t num_free() {
    std::lock_guard<std::mutex> g(mu_);
    return (int32_t)free_.size();
  }

  // -1 for an id outside the pool
  int32_t refcount(int32_t id) {
    std::lock_guard<std::mutex> g(mu_);
    return valid(id) ? refs_[id] : -1;
  }

  // n fresh blocks with count 1, or none at all (returns false) if fewer are free
  bool alloc(int32_t n, int32_t* ids) {
    std::lock_guard<std::mutex> g(mu_);
    if (n < 0 || (size_t)n > free_.size()) return false;
    for (int32_t i = 0; i < n; ++i) {
      const int32_t b = free_.back();
      free_.pop_back();
      refs_[b] = 1;
      ids[i] = b;
    }
    return true;
  }

  // one more holder for each block; all must be live, else nothing changes
  bool share(const int32_t* ids, int32_t n) {
    std::lock_guard<std::mutex> g(mu_);
    for (int32_t i = 0; i < n; ++i)
      if (!valid(ids[i]) || refs_[ids[i]] <= 0) return false;
    for (int32_t i = 0; i < n; ++i) ++refs_[ids[i]];
    return true;
  }

  // one holder fewer for each block; a block whose count reaches 0 is free
  // again.  All must be live with enough holders (an id may repeat), else
  // nothing changes.
  bool release(const int32_t* ids, int32_t n) {
    std::lock_guard<std::mutex> g(mu_);
    std::vector<int32_t> dec;
    for (int32_t i = 0; i < n; ++i) {
      if (!valid(ids[i])) return false;
      int32_t seen = 0;
      for (int32_t j = 0; j < i; ++j) seen += ids[j] == ids[i];
      if (refs_[ids[i]] <= seen) return false;
    }
    for (int32_t i = 0; i < n; ++i)
      if (--refs_[ids[i]] == 0) free_.push_back(ids[i]);
    return true;
  }

  // Before writing into block `id`: if it is shared, take a fresh block for
  // the writer (the caller copies id -> new_id on the device) and give up one
  // hold on id; if it is private, write in place.  Returns false if id is not
  // live, or no block is free for the copy (then nothing changes).
  bool copy_on_write(int32_t id, int32_t* new_id, bool* must_copy) {
    std::lock_guard<std::mutex> g(mu_);
    if (!valid(id) || refs_[id] <= 0) return false;
    if (refs_[id] == 1) {
      *new_id = id;
      *must_copy = false;
      return true;
    }
    if (free_.empty()) return false;
    const int32_t b = free_.back();
    free_.pop_back();
    refs_[b] = 1;
    --refs_[id];
    *new_id = b;
    *must_copy = true;
    return true;
  }

 private:
  bool valid(int32_t id) const { return id >= 0 && (size_t)id < refs_.size(); }
  std::mutex mu_;
  std::vector<int32_t> refs_;
  std::vector<int32_t> free_;
};

}  // namespace pkv
