// Host-side block pool and continuous-batching planner (include/deltakv_pool.h).  Plain C++: no CUDA calls,
// no device memory.  The serving engine on the DeltaKV pages keeps memory management apart from kernel
// execution (summary (en) §4 "Sparse-vLLM Engine"); this file is that management for the paged cache layout
// of deltakv.h, and the scheduler that turns queued requests into compress / decode batches.
#include <algorithm>
#include <deque>
#include <new>
#include <vector>

#include "../../include/deltakv_pool.h"

namespace {

// 64-bit mixing generator (the splitmix64 output function over a Weyl sequence); used only to draw the
// seeded placement order of free blocks.
struct Mix64 {
  uint64_t s;
  uint64_t next() {
    uint64_t z = (s += 0x9E3779B97F4A7C15ull);
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
  }
};

int32_t blocks_for(int64_t len, int32_t R) { return static_cast<int32_t>((len + R - 1) / R); }

}  // namespace

struct dkv_pool {
  int32_t num_blocks = 0, R = 0, max_seqs = 0, max_bps = 0;
  std::vector<int32_t> free_blocks;  // the back is handed out next
  std::vector<int32_t> free_slots;   // closed sequence ids, the back is reused next
  std::vector<std::vector<int32_t>> table;
  std::vector<int32_t> len;
  std::vector<uint8_t> is_open;

  bool valid_seq(int32_t s) const { return s >= 0 && s < max_seqs && is_open[s]; }
};

struct dkv_batcher {
  struct Req {
    int64_t id;
    int32_t prompt, max_new;
    int32_t generated = 0;  // tokens generated so far (a preempted request keeps its count)
    int32_t seq = -1;
    bool fresh = false;     // admitted by the current plan: its compress entry is the whole prefix
  };
  dkv_pool* pool = nullptr;
  int32_t max_prefill = 0, max_batch = 0;
  std::deque<Req> waiting;
  std::vector<Req> running;  // admission order
  int64_t finished = 0;
  bool planned = false;      // a plan is waiting for its commit
};

extern "C" {

dkv_status deltakv_pool_create(int32_t num_blocks, int32_t block_tokens, int32_t max_seqs, int32_t max_blocks_per_seq,
                               uint64_t seed, dkv_pool** out) {
  if (out == nullptr || num_blocks <= 0 || block_tokens <= 0 || max_seqs <= 0 || max_blocks_per_seq <= 0)
    return DKV_ERR_INVALID_ARG;
  dkv_pool* p = new (std::nothrow) dkv_pool;
  if (p == nullptr) return DKV_ERR_INVALID_ARG;
  p->num_blocks = num_blocks;
  p->R = block_tokens;
  p->max_seqs = max_seqs;
  p->max_bps = max_blocks_per_seq;
  std::vector<int32_t> order(num_blocks);
  for (int32_t i = 0; i < num_blocks; ++i) order[i] = i;
  if (seed != 0) {  // Fisher-Yates with the mixing generator
    Mix64 g{seed};
    for (int32_t i = num_blocks - 1; i > 0; --i) std::swap(order[i], order[g.next() % static_cast<uint64_t>(i + 1)]);
  }
  p->free_blocks.assign(order.rbegin(), order.rend());  // order[0] is handed out first
  p->free_slots.resize(max_seqs);
  for (int32_t i = 0; i < max_seqs; ++i) p->free_slots[i] = max_seqs - 1 - i;
  p->table.resize(max_seqs);
  p->len.assign(max_seqs, 0);
  p->is_open.assign(max_seqs, 0);
  *out = p;
  return DKV_OK;
}

void deltakv_pool_destroy(dkv_pool* pool) { delete pool; }

int32_t deltakv_pool_num_free(const dkv_pool* pool) {
  return pool == nullptr ? 0 : static_cast<int32_t>(pool->free_blocks.size());
}

dkv_status deltakv_pool_open(dkv_pool* p, int32_t* seq) {
  if (p == nullptr || seq == nullptr) return DKV_ERR_INVALID_ARG;
  if (p->free_slots.empty()) return DKV_ERR_OUT_OF_BLOCKS;
  const int32_t s = p->free_slots.back();
  p->free_slots.pop_back();
  p->is_open[s] = 1;
  p->len[s] = 0;
  p->table[s].clear();
  *seq = s;
  return DKV_OK;
}

dkv_status deltakv_pool_grow(dkv_pool* p, int32_t seq, int32_t new_len) {
  if (p == nullptr || !p->valid_seq(seq) || new_len < p->len[seq]) return DKV_ERR_INVALID_ARG;
  const int32_t want = blocks_for(new_len, p->R);
  const int32_t have = static_cast<int32_t>(p->table[seq].size());
  const int32_t need = want - have;
  if (want > p->max_bps || need > static_cast<int32_t>(p->free_blocks.size())) return DKV_ERR_OUT_OF_BLOCKS;
  for (int32_t i = 0; i < need; ++i) {
    p->table[seq].push_back(p->free_blocks.back());
    p->free_blocks.pop_back();
  }
  p->len[seq] = new_len;
  return DKV_OK;
}

dkv_status deltakv_pool_close(dkv_pool* p, int32_t seq) {
  if (p == nullptr || !p->valid_seq(seq)) return DKV_ERR_INVALID_ARG;
  std::vector<int32_t>& t = p->table[seq];
  for (auto it = t.rbegin(); it != t.rend(); ++it) p->free_blocks.push_back(*it);  // first block reused first
  t.clear();
  p->len[seq] = 0;
  p->is_open[seq] = 0;
  p->free_slots.push_back(seq);
  return DKV_OK;
}

dkv_status deltakv_pool_seq_info(const dkv_pool* p, int32_t seq, int32_t* len, int32_t* blocks) {
  if (p == nullptr || !p->valid_seq(seq)) return DKV_ERR_INVALID_ARG;
  if (len) *len = p->len[seq];
  if (blocks) *blocks = static_cast<int32_t>(p->table[seq].size());
  return DKV_OK;
}

dkv_status deltakv_pool_block_tables(const dkv_pool* p, const int32_t* seqs, int32_t n, int32_t max_blocks,
                                     int32_t* out) {
  if (p == nullptr || n < 0 || max_blocks <= 0 || (n > 0 && (seqs == nullptr || out == nullptr)))
    return DKV_ERR_INVALID_ARG;
  for (int32_t i = 0; i < n; ++i)
    if (!p->valid_seq(seqs[i]) || static_cast<int32_t>(p->table[seqs[i]].size()) > max_blocks)
      return DKV_ERR_INVALID_ARG;
  for (int32_t i = 0; i < n; ++i) {
    const std::vector<int32_t>& t = p->table[seqs[i]];
    int32_t* row = out + static_cast<int64_t>(i) * max_blocks;
    std::copy(t.begin(), t.end(), row);
    std::fill(row + t.size(), row + max_blocks, -1);
  }
  return DKV_OK;
}

dkv_status deltakv_batcher_create(dkv_pool* pool, int32_t max_prefill_tokens, int32_t max_batch, dkv_batcher** out) {
  if (pool == nullptr || out == nullptr || max_prefill_tokens <= 0 || max_batch <= 0) return DKV_ERR_INVALID_ARG;
  dkv_batcher* b = new (std::nothrow) dkv_batcher;
  if (b == nullptr) return DKV_ERR_INVALID_ARG;
  b->pool = pool;
  b->max_prefill = max_prefill_tokens;
  b->max_batch = max_batch;
  *out = b;
  return DKV_OK;
}

void deltakv_batcher_destroy(dkv_batcher* b) { delete b; }

dkv_status deltakv_batcher_submit(dkv_batcher* b, int64_t id, int32_t prompt_len, int32_t max_new_tokens) {
  if (b == nullptr || prompt_len <= 0 || max_new_tokens <= 0) return DKV_ERR_INVALID_ARG;
  // the longest context a request reaches is prompt + max_new - 1 tokens; it must fit one sequence and the pool
  const int64_t longest = static_cast<int64_t>(prompt_len) + max_new_tokens - 1;
  const int64_t blocks = (longest + b->pool->R - 1) / b->pool->R;
  if (blocks > b->pool->max_bps || blocks > b->pool->num_blocks) return DKV_ERR_INVALID_ARG;
  for (const auto& r : b->waiting)
    if (r.id == id) return DKV_ERR_INVALID_ARG;
  for (const auto& r : b->running)
    if (r.id == id) return DKV_ERR_INVALID_ARG;
  dkv_batcher::Req r;
  r.id = id;
  r.prompt = prompt_len;
  r.max_new = max_new_tokens;
  b->waiting.push_back(r);
  return DKV_OK;
}

dkv_status deltakv_batcher_plan(dkv_batcher* b, dkv_step_plan* plan) {
  if (b == nullptr || plan == nullptr || b->planned) return DKV_ERR_INVALID_ARG;
  if (plan->comp_req == nullptr || plan->comp_seq == nullptr || plan->cu_new == nullptr ||
      plan->start_pos == nullptr || plan->comp_from == nullptr || plan->dec_req == nullptr ||
      plan->dec_seq == nullptr || plan->context_len == nullptr)
    return DKV_ERR_INVALID_ARG;
  dkv_pool* p = b->pool;
  int32_t preempted = 0;
  // 1. every running request reserves room for the token generated by the previous step; out of blocks, the
  //    most recently admitted one is preempted (recomputed later from its prompt and generated tokens)
  for (size_t i = 0; i < b->running.size();) {
    dkv_batcher::Req& r = b->running[i];
    r.fresh = false;
    const int32_t next_len = r.prompt + r.generated;  // cache holds prompt + generated - 1 tokens
    const dkv_status st = deltakv_pool_grow(p, r.seq, next_len);
    if (st == DKV_OK) {
      ++i;
      continue;
    }
    if (st != DKV_ERR_OUT_OF_BLOCKS) return st;
    dkv_batcher::Req victim = b->running.back();
    b->running.pop_back();
    deltakv_pool_close(p, victim.seq);
    victim.seq = -1;
    b->waiting.push_front(victim);
    ++preempted;
    // if the victim was request i itself, the loop ends (i == size); otherwise request i retries
  }
  // 2. first come, first served admission within the prefill budget, the batch limit and the pool
  int32_t prefill_rows = 0;
  while (!b->waiting.empty() && static_cast<int32_t>(b->running.size()) < b->max_batch) {
    dkv_batcher::Req r = b->waiting.front();
    const int32_t n = r.prompt + r.generated;  // a recomputed request re-supplies its generated tokens too
    if (prefill_rows > 0 && prefill_rows + n > b->max_prefill) break;
    int32_t seq = -1;
    if (deltakv_pool_open(p, &seq) != DKV_OK) break;
    if (deltakv_pool_grow(p, seq, n) != DKV_OK) {
      deltakv_pool_close(p, seq);
      break;
    }
    b->waiting.pop_front();
    r.seq = seq;
    r.fresh = true;
    b->running.push_back(r);
    prefill_rows += n;
  }
  // 3. emit: compress appends / prefixes and the decode of every running request, in admission order
  int32_t nc = 0, row = 0;
  plan->cu_new[0] = 0;
  for (const dkv_batcher::Req& r : b->running) {
    int32_t len = 0;
    deltakv_pool_seq_info(p, r.seq, &len, nullptr);
    const int32_t n = r.fresh ? len : 1;
    plan->comp_req[nc] = r.id;
    plan->comp_seq[nc] = r.seq;
    plan->start_pos[nc] = len - n;
    plan->comp_from[nc] = len - n;
    row += n;
    plan->cu_new[nc + 1] = row;
    plan->dec_req[nc] = r.id;
    plan->dec_seq[nc] = r.seq;
    plan->context_len[nc] = len;
    ++nc;
  }
  plan->num_compress = nc;
  plan->num_decode = nc;
  plan->num_preempted = preempted;
  b->planned = true;
  return DKV_OK;
}

dkv_status deltakv_batcher_commit(dkv_batcher* b, int64_t* finished, int32_t* num_finished) {
  if (b == nullptr || !b->planned) return DKV_ERR_INVALID_ARG;
  int32_t nf = 0;
  std::vector<dkv_batcher::Req> keep;
  keep.reserve(b->running.size());
  for (dkv_batcher::Req& r : b->running) {
    r.generated += 1;
    r.fresh = false;
    if (r.generated >= r.max_new) {
      deltakv_pool_close(b->pool, r.seq);
      if (finished != nullptr) finished[nf] = r.id;
      ++nf;
      ++b->finished;
    } else {
      keep.push_back(r);
    }
  }
  b->running.swap(keep);
  if (num_finished != nullptr) *num_finished = nf;
  b->planned = false;
  return DKV_OK;
}

dkv_status deltakv_batcher_counts(const dkv_batcher* b, int32_t* waiting, int32_t* running, int64_t* finished) {
  if (b == nullptr) return DKV_ERR_INVALID_ARG;
  if (waiting) *waiting = static_cast<int32_t>(b->waiting.size());
  if (running) *running = static_cast<int32_t>(b->running.size());
  if (finished) *finished = b->finished;
  return DKV_OK;
}

}  // extern "C"
