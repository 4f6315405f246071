// pa_alloc.cpp -- host block allocator of the paged KV cache.
//
// zingnex.cn, "vLLM与PagedAttention深度剖析", section 3.2: blocks are taken
// only when a token crosses into a new block (item 1), a sequence's blocks
// need not be contiguous and are found through its block table (item 2),
// sharers of a block copy it before writing (item 3), and freed blocks are
// reused from a pool instead of new device allocations (item 4).  jsqmd.com
// "vLLM-v0.11.0性能实测" section 4.2 adds sharing of a common prefix.
//
// The free list is a stack (last freed, first reused); reference counts make
// sharing and copy-on-write explicit.  Everything here is host memory.
#include <cstdint>
#include <unordered_map>
#include <vector>

#include "pa.h"

struct pa_alloc {
  int32_t num_blocks = 0;
  int32_t block_size = 0;
  std::vector<int32_t> free_stack;  // back() is the next block handed out
  std::vector<int32_t> ref;
  struct Seq {
    std::vector<int32_t> blocks;
    int64_t len = 0;
  };
  std::unordered_map<int32_t, Seq> seqs;

  int32_t take() {
    const int32_t b = free_stack.back();
    free_stack.pop_back();
    ref[b] = 1;
    return b;
  }
  void release(int32_t b) {
    if (--ref[b] == 0) free_stack.push_back(b);
  }
  int64_t blocks_for(int64_t tokens) const { return (tokens + block_size - 1) / block_size; }
};

extern "C" {

pa_alloc* pa_alloc_create(int32_t num_blocks, int32_t block_size, const int32_t* order) {
  if (num_blocks <= 0 || block_size <= 0) return nullptr;
  auto* a = new pa_alloc;
  a->num_blocks = num_blocks;
  a->block_size = block_size;
  a->ref.assign(num_blocks, 0);
  a->free_stack.resize(num_blocks);
  std::vector<char> seen(num_blocks, 0);
  for (int32_t i = 0; i < num_blocks; ++i) {
    const int32_t b = order ? order[i] : i;
    if (b < 0 || b >= num_blocks || seen[b]) {
      delete a;
      return nullptr;
    }
    seen[b] = 1;
    a->free_stack[num_blocks - 1 - i] = b;  // order[0] on top
  }
  return a;
}

void pa_alloc_destroy(pa_alloc* a) { delete a; }

pa_status pa_alloc_extend(pa_alloc* a, int32_t seq, int32_t num_tokens) {
  if (!a || num_tokens < 0) return PA_ERR_INVALID_ARG;
  auto it = a->seqs.find(seq);
  if (it == a->seqs.end()) return PA_ERR_INVALID_ARG;
  auto& s = it->second;
  const int64_t need = a->blocks_for(s.len + num_tokens) - (int64_t)s.blocks.size();
  if (need > (int64_t)a->free_stack.size()) return PA_ERR_OOM;
  for (int64_t i = 0; i < need; ++i) s.blocks.push_back(a->take());
  s.len += num_tokens;
  return PA_OK;
}

pa_status pa_alloc_add_seq(pa_alloc* a, int32_t seq, int32_t num_tokens) {
  if (!a || num_tokens < 0) return PA_ERR_INVALID_ARG;
  if (a->seqs.count(seq)) return PA_ERR_INVALID_ARG;
  if (a->blocks_for(num_tokens) > (int64_t)a->free_stack.size()) return PA_ERR_OOM;
  a->seqs.emplace(seq, pa_alloc::Seq{});
  return pa_alloc_extend(a, seq, num_tokens);
}

pa_status pa_alloc_fork(pa_alloc* a, int32_t parent, int32_t child) {
  if (!a) return PA_ERR_INVALID_ARG;
  auto it = a->seqs.find(parent);
  if (it == a->seqs.end() || a->seqs.count(child)) return PA_ERR_INVALID_ARG;
  pa_alloc::Seq c = it->second;
  for (int32_t b : c.blocks) ++a->ref[b];
  a->seqs.emplace(child, std::move(c));
  return PA_OK;
}

pa_status pa_alloc_free_seq(pa_alloc* a, int32_t seq) {
  if (!a) return PA_ERR_INVALID_ARG;
  auto it = a->seqs.find(seq);
  if (it == a->seqs.end()) return PA_ERR_INVALID_ARG;
  const auto& blocks = it->second.blocks;
  for (auto r = blocks.rbegin(); r != blocks.rend(); ++r) a->release(*r);
  a->seqs.erase(it);
  return PA_OK;
}

pa_status pa_alloc_append_slots(pa_alloc* a, const int32_t* seqs, int32_t n, int32_t* slot_out,
                                int32_t* pairs_out, int32_t* num_pairs_out) {
  if (!a || n < 0 || (n > 0 && (!seqs || !slot_out || !pairs_out || !num_pairs_out)))
    return PA_ERR_INVALID_ARG;
  // Dry run: count fresh blocks, tracking reference drops of shared last
  // blocks within the batch, so the call is all-or-nothing.
  std::unordered_map<int32_t, int32_t> ref_drop;
  int64_t need = 0;
  for (int32_t i = 0; i < n; ++i) {
    auto it = a->seqs.find(seqs[i]);
    if (it == a->seqs.end()) return PA_ERR_INVALID_ARG;
    for (int32_t j = 0; j < i; ++j)
      if (seqs[j] == seqs[i]) return PA_ERR_INVALID_ARG;  // one token per sequence per call
    const auto& s = it->second;
    if (s.len % a->block_size == 0) {
      ++need;
    } else {
      const int32_t last = s.blocks.back();
      if (a->ref[last] - ref_drop[last] > 1) {
        ++need;
        ++ref_drop[last];
      }
    }
  }
  if (need > (int64_t)a->free_stack.size()) return PA_ERR_OOM;
  int32_t np = 0;
  for (int32_t i = 0; i < n; ++i) {
    auto& s = a->seqs[seqs[i]];
    const int32_t off = (int32_t)(s.len % a->block_size);
    int32_t b;
    if (off == 0) {
      b = a->take();
      s.blocks.push_back(b);
    } else {
      b = s.blocks.back();
      if (a->ref[b] > 1) {
        const int32_t nb = a->take();
        pairs_out[2 * np] = b;
        pairs_out[2 * np + 1] = nb;
        ++np;
        a->release(b);
        s.blocks.back() = nb;
        b = nb;
      }
    }
    slot_out[i] = b * a->block_size + off;
    s.len += 1;
  }
  *num_pairs_out = np;
  return PA_OK;
}

pa_status pa_alloc_block_tables(const pa_alloc* a, const int32_t* seqs, int32_t n,
                                int32_t max_blocks_per_seq, int32_t* tables_out,
                                int32_t* lens_out) {
  if (!a || n < 0 || max_blocks_per_seq < 0 || (n > 0 && (!seqs || !tables_out || !lens_out)))
    return PA_ERR_INVALID_ARG;
  for (int32_t i = 0; i < n; ++i) {
    auto it = a->seqs.find(seqs[i]);
    if (it == a->seqs.end()) return PA_ERR_INVALID_ARG;
    const auto& s = it->second;
    if ((int64_t)s.blocks.size() > max_blocks_per_seq) return PA_ERR_INVALID_ARG;
    int32_t* row = tables_out + (int64_t)i * max_blocks_per_seq;
    for (int32_t j = 0; j < max_blocks_per_seq; ++j)
      row[j] = j < (int32_t)s.blocks.size() ? s.blocks[j] : -1;
    lens_out[i] = (int32_t)s.len;
  }
  return PA_OK;
}

int32_t pa_alloc_num_free(const pa_alloc* a) { return a ? (int32_t)a->free_stack.size() : -1; }

int32_t pa_alloc_refcount(const pa_alloc* a, int32_t block) {
  if (!a || block < 0 || block >= a->num_blocks) return -1;
  return a->ref[block];
}

}  // extern "C"
