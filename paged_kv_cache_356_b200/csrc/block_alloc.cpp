// pa_block_alloc: host-side ref-counted free-page pool and per-sequence block
// tables -- the control plane of the paged KV cache.
//
// PagedAttention Internals, "2. The Dynamic Block Table": one table per
// sequence maps logical blocks to physical pages taken on demand from a global
// free-page pool.  "Implementation: Custom Block Manager Simulation in Python":
// ceil(n / bs) pages per sequence, an out-of-memory failure checked before any
// page is taken, pages taken from the front of the pool and returned to its
// back in table order when their count reaches zero, a fresh page at count 1,
// freeing an unknown sequence is a no-op.  "Copy-on-Write and Prefix Sharing"
// (and the glossary's "Copy-on-Write Memory Forking"): shared pages carry a
// reference count, and a page is duplicated only when a sequence writes into
// it while others still hold it.
//
// The pool is a fixed ring of num_blocks ids (it can never hold more), so
// taking from the front and returning to the back are O(1).
#include <algorithm>
#include <climits>
#include <unordered_map>
#include <vector>

#include "pa_internal.h"

struct pa_block_alloc {
  int32_t num_blocks = 0;
  int32_t block_size = 0;
  std::vector<int32_t> ring;  // free pool, front at `head`, `count` ids
  int64_t head = 0;
  int64_t count = 0;
  std::vector<int32_t> refs;
  struct Seq {
    std::vector<int32_t> pages;
    int64_t tokens = 0;
    // Change log for pa_block_alloc_table_updates: table entries changed since
    // the sequence was last exported there, or the whole table.
    std::vector<int32_t> changed;
    bool whole = true;
    int32_t row = -1;  // the export row the log is relative to
    void log(int32_t logical) {
      if (whole) return;
      if (changed.size() >= pages.size()) {  // more entries logged than held: export it whole
        whole = true;
        changed.clear();
        return;
      }
      changed.push_back(logical);
    }
  };
  std::unordered_map<int64_t, Seq> seqs;
  // Rows of the incremental export: the sequence each row was last exported
  // for (kNoOwner: unknown contents) and how many leading entries it holds.
  static constexpr int64_t kNoOwner = INT64_MIN;
  std::vector<int64_t> row_owner;
  std::vector<int32_t> row_len;
  int32_t rows_width = -1;  // max_blocks_per_seq of the recorded rows

  int32_t take_front() {
    int32_t page = ring[head];
    head = (head + 1) % num_blocks;
    --count;
    refs[page] = 1;
    return page;
  }
  void release(int32_t page) {
    if (--refs[page] == 0) {
      ring[(head + count) % num_blocks] = page;
      ++count;
    }
  }
};

using pa::fail;

extern "C" {

pa_status pa_block_alloc_create(int32_t num_blocks, int32_t block_size,
                                const int32_t* initial_free_order, pa_block_alloc** out) {
  if (!out) return fail(PA_ERR_INVALID, "pa_block_alloc_create: out is NULL");
  *out = nullptr;
  if (num_blocks < 0 || block_size <= 0)
    return fail(PA_ERR_INVALID, "pa_block_alloc_create: num_blocks=%d block_size=%d", num_blocks,
                block_size);
  auto* a = new pa_block_alloc();
  a->num_blocks = num_blocks;
  a->block_size = block_size;
  a->ring.resize(num_blocks > 0 ? num_blocks : 1);
  a->refs.assign(num_blocks, 0);
  if (initial_free_order) {
    std::vector<char> seen(num_blocks, 0);
    for (int32_t i = 0; i < num_blocks; ++i) {
      int32_t p = initial_free_order[i];
      if (p < 0 || p >= num_blocks || seen[p]) {
        delete a;
        return fail(PA_ERR_INVALID, "pa_block_alloc_create: initial_free_order is not a permutation");
      }
      seen[p] = 1;
      a->ring[i] = p;
    }
  } else {
    for (int32_t i = 0; i < num_blocks; ++i) a->ring[i] = i;
  }
  a->count = num_blocks;
  *out = a;
  return PA_OK;
}

void pa_block_alloc_destroy(pa_block_alloc* a) { delete a; }

pa_status pa_block_alloc_allocate_sequence(pa_block_alloc* a, int64_t seq, int64_t num_tokens) {
  if (!a) return fail(PA_ERR_INVALID, "allocate_sequence: NULL handle");
  if (num_tokens < 0) return fail(PA_ERR_INVALID, "allocate_sequence: num_tokens=%lld", (long long)num_tokens);
  if (a->seqs.count(seq)) return fail(PA_ERR_INVALID, "allocate_sequence: sequence %lld exists", (long long)seq);
  int64_t need = (num_tokens + a->block_size - 1) / a->block_size;
  if (need > a->count)
    return fail(PA_ERR_OOM, "allocate_sequence: %lld pages needed, %lld free", (long long)need,
                (long long)a->count);
  auto& s = a->seqs[seq];
  s.pages.reserve(need);
  for (int64_t i = 0; i < need; ++i) s.pages.push_back(a->take_front());
  s.tokens = num_tokens;
  return PA_OK;
}

pa_status pa_block_alloc_append_token(pa_block_alloc* a, int64_t seq, int64_t* slot_out,
                                      int32_t* cow_src, int32_t* cow_dst) {
  if (!a) return fail(PA_ERR_INVALID, "append_token: NULL handle");
  auto it = a->seqs.find(seq);
  if (it == a->seqs.end()) return fail(PA_ERR_NOT_FOUND, "append_token: unknown sequence %lld", (long long)seq);
  auto& s = it->second;
  const int64_t pos = s.tokens;
  const int64_t logical = pos / a->block_size;
  const int64_t offset = pos % a->block_size;
  int32_t src = -1, dst = -1;
  if (offset == 0) {
    if (a->count == 0) return fail(PA_ERR_OOM, "append_token: no free page for the next block");
    s.pages.push_back(a->take_front());
    s.log((int32_t)logical);
  } else if (a->refs[s.pages[logical]] > 1) {
    if (!cow_src || !cow_dst)
      return fail(PA_ERR_INVALID, "append_token: page %d is shared but cow_src/cow_dst are NULL",
                  s.pages[logical]);
    if (a->count == 0) return fail(PA_ERR_OOM, "append_token: no free page for the copy-on-write fork");
    src = s.pages[logical];
    dst = a->take_front();
    a->release(src);
    s.pages[logical] = dst;
    s.log((int32_t)logical);
  }
  s.tokens = pos + 1;
  if (slot_out) *slot_out = (int64_t)s.pages[logical] * a->block_size + offset;
  if (cow_src) *cow_src = src;
  if (cow_dst) *cow_dst = dst;
  return PA_OK;
}

pa_status pa_block_alloc_append_tokens(pa_block_alloc* a, const int64_t* seqs, int32_t n, int64_t* slots_out,
                                       int32_t* cow_src, int32_t* cow_dst, int32_t* n_done) {
  if (n_done) *n_done = 0;
  if (!a || n < 0 || (n > 0 && (!seqs || !cow_src || !cow_dst)))
    return fail(PA_ERR_INVALID, "append_tokens: bad argument");
  for (int32_t i = 0; i < n; ++i) {
    const pa_status st =
        pa_block_alloc_append_token(a, seqs[i], slots_out ? slots_out + i : nullptr, cow_src + i, cow_dst + i);
    if (st != PA_OK) return st;  // that append changed nothing; the earlier ones stand
    if (n_done) *n_done = i + 1;
  }
  return PA_OK;
}

pa_status pa_block_alloc_fork(pa_block_alloc* a, int64_t parent, int64_t child) {
  if (!a) return fail(PA_ERR_INVALID, "fork: NULL handle");
  auto it = a->seqs.find(parent);
  if (it == a->seqs.end()) return fail(PA_ERR_NOT_FOUND, "fork: unknown parent %lld", (long long)parent);
  if (a->seqs.count(child)) return fail(PA_ERR_INVALID, "fork: sequence %lld exists", (long long)child);
  pa_block_alloc::Seq copy = it->second;  // copy before inserting (rehash may move `it`)
  copy.changed.clear();
  copy.whole = true;  // a new sequence: its whole table is exported
  for (int32_t p : copy.pages) ++a->refs[p];
  a->seqs.emplace(child, std::move(copy));
  return PA_OK;
}

pa_status pa_block_alloc_free_sequence(pa_block_alloc* a, int64_t seq) {
  if (!a) return fail(PA_ERR_INVALID, "free_sequence: NULL handle");
  auto it = a->seqs.find(seq);
  if (it == a->seqs.end()) return PA_OK;
  for (int32_t p : it->second.pages) a->release(p);
  a->seqs.erase(it);
  return PA_OK;
}

pa_status pa_block_alloc_slot_mapping(const pa_block_alloc* a, int64_t seq, int64_t start,
                                      int64_t count, int64_t* out) {
  if (!a || (!out && count > 0)) return fail(PA_ERR_INVALID, "slot_mapping: NULL argument");
  auto it = a->seqs.find(seq);
  if (it == a->seqs.end()) return fail(PA_ERR_NOT_FOUND, "slot_mapping: unknown sequence %lld", (long long)seq);
  const auto& s = it->second;
  if (start < 0 || count < 0 || start + count > s.tokens)
    return fail(PA_ERR_INVALID, "slot_mapping: positions [%lld, %lld) outside [0, %lld)", (long long)start,
                (long long)(start + count), (long long)s.tokens);
  const int64_t bs = a->block_size;
  for (int64_t i = 0; i < count; ++i) {
    const int64_t pos = start + i;
    out[i] = (int64_t)s.pages[pos / bs] * bs + pos % bs;
  }
  return PA_OK;
}

pa_status pa_block_alloc_block_table(const pa_block_alloc* a, int64_t seq, int32_t* out, int32_t cap,
                                     int32_t* n_out) {
  if (!a) return fail(PA_ERR_INVALID, "block_table: NULL handle");
  auto it = a->seqs.find(seq);
  if (it == a->seqs.end()) return fail(PA_ERR_NOT_FOUND, "block_table: unknown sequence %lld", (long long)seq);
  const auto& pages = it->second.pages;
  if (n_out) *n_out = (int32_t)pages.size();
  if ((int64_t)pages.size() > cap || (!out && !pages.empty()))
    return fail(PA_ERR_INVALID, "block_table: %zu entries, capacity %d", pages.size(), cap);
  for (size_t i = 0; i < pages.size(); ++i) out[i] = pages[i];
  return PA_OK;
}

pa_status pa_block_alloc_block_tables(const pa_block_alloc* a, const int64_t* seqs, int32_t n, int32_t* out,
                                      int32_t max_blocks_per_seq, int32_t pad, int32_t* context_lens_out) {
  if (!a || n < 0 || max_blocks_per_seq < 0 || (n > 0 && (!seqs || !out)))
    return fail(PA_ERR_INVALID, "block_tables: bad argument");
  for (int32_t i = 0; i < n; ++i) {
    auto it = a->seqs.find(seqs[i]);
    if (it == a->seqs.end())
      return fail(PA_ERR_NOT_FOUND, "block_tables: unknown sequence %lld", (long long)seqs[i]);
    const auto& pages = it->second.pages;
    if ((int64_t)pages.size() > max_blocks_per_seq)
      return fail(PA_ERR_INVALID, "block_tables: sequence %lld holds %zu pages > %d", (long long)seqs[i],
                  pages.size(), max_blocks_per_seq);
    int32_t* row = out + (int64_t)i * max_blocks_per_seq;
    size_t j = 0;
    for (; j < pages.size(); ++j) row[j] = pages[j];
    for (; j < (size_t)max_blocks_per_seq; ++j) row[j] = pad;
    if (context_lens_out) context_lens_out[i] = (int32_t)it->second.tokens;
  }
  return PA_OK;
}

int64_t pa_block_alloc_num_tokens(const pa_block_alloc* a, int64_t seq) {
  if (!a) return -1;
  auto it = a->seqs.find(seq);
  return it == a->seqs.end() ? -1 : it->second.tokens;
}

int32_t pa_block_alloc_num_free(const pa_block_alloc* a) { return a ? (int32_t)a->count : -1; }

int32_t pa_block_alloc_num_sequences(const pa_block_alloc* a) { return a ? (int32_t)a->seqs.size() : -1; }

int32_t pa_block_alloc_ref_count(const pa_block_alloc* a, int32_t page) {
  if (!a || page < 0 || page >= a->num_blocks) return -1;
  return a->refs[page];
}

pa_status pa_block_alloc_free_pool(const pa_block_alloc* a, int32_t* out, int32_t cap, int32_t* n_out) {
  if (!a) return fail(PA_ERR_INVALID, "free_pool: NULL handle");
  if (n_out) *n_out = (int32_t)a->count;
  if (a->count > cap || (!out && a->count > 0))
    return fail(PA_ERR_INVALID, "free_pool: %lld entries, capacity %d", (long long)a->count, cap);
  for (int64_t i = 0; i < a->count; ++i) out[i] = a->ring[(a->head + i) % a->num_blocks];
  return PA_OK;
}

pa_status pa_block_alloc_stats(const pa_block_alloc* a, double alarm_free_fraction, pa_pool_stats* out) {
  if (!a || !out) return fail(PA_ERR_INVALID, "stats: NULL argument");
  const int64_t bs = a->block_size;
  // Filled slots per page: the most any holder has stored in it.
  std::vector<int32_t> filled(a->num_blocks, 0);
  pa_pool_stats st{};
  st.num_blocks = a->num_blocks;
  st.block_size = a->block_size;
  st.free_pages = (int32_t)a->count;
  st.num_sequences = (int32_t)a->seqs.size();
  for (const auto& kv : a->seqs) {
    const auto& sq = kv.second;
    st.logical_tokens += sq.tokens;
    for (size_t i = 0; i < sq.pages.size(); ++i) {
      const int64_t n = std::min<int64_t>(bs, sq.tokens - (int64_t)i * bs);
      int32_t& f = filled[sq.pages[i]];
      if (n > f) f = (int32_t)n;
    }
  }
  for (int32_t p = 0; p < a->num_blocks; ++p) {
    if (a->refs[p] > 0) ++st.used_pages;
    if (a->refs[p] > 1) ++st.shared_pages;
    st.physical_tokens += filled[p];
  }
  st.waste_slots = (int64_t)st.used_pages * bs - st.physical_tokens;
  st.waste_fraction = st.used_pages > 0 ? (double)st.waste_slots / (double)((int64_t)st.used_pages * bs) : 0.0;
  st.free_fraction = a->num_blocks > 0 ? (double)st.free_pages / (double)a->num_blocks : 0.0;
  st.low_free_alarm = a->num_blocks > 0 && st.free_fraction < alarm_free_fraction;
  *out = st;
  return PA_OK;
}

pa_status pa_block_alloc_prefix_plan(const pa_block_alloc* a, const int64_t* seqs, int32_t n, int32_t group_size,
                                     int32_t* first_partition, int32_t* chunks, int32_t* members, int32_t* num_chunks,
                                     int32_t* num_members, int32_t* max_shared_partitions,
                                     int32_t* min_shared_partitions) {
  if (!a || n < 0 || (n > 0 && (!seqs || !first_partition || !chunks || !members)) || !num_chunks ||
      !num_members || !max_shared_partitions || !min_shared_partitions)
    return fail(PA_ERR_INVALID, "prefix_plan: bad argument");
  if (group_size < 1 || group_size > PA_PREFIX_QUERIES_PER_CTA)
    return fail(PA_ERR_INVALID, "prefix_plan: group_size %d outside [1, %d]", group_size, PA_PREFIX_QUERIES_PER_CTA);
  std::vector<const pa_block_alloc::Seq*> batch(n);
  for (int32_t i = 0; i < n; ++i) {
    auto it = a->seqs.find(seqs[i]);
    if (it == a->seqs.end()) return fail(PA_ERR_NOT_FOUND, "prefix_plan: unknown sequence %lld", (long long)seqs[i]);
    batch[i] = &it->second;
    first_partition[i] = 0;
  }
  // Candidate groups: sequences whose first page is the same shared page, in batch order.
  std::unordered_map<int32_t, std::vector<int32_t>> by_first;
  std::vector<int32_t> order;
  for (int32_t i = 0; i < n; ++i) {
    const auto& pages = batch[i]->pages;
    if (pages.empty() || a->refs[pages[0]] < 2) continue;
    auto& v = by_first[pages[0]];
    if (v.empty()) order.push_back(pages[0]);
    v.push_back(i);
  }
  const int32_t per_chunk = std::max(1, PA_PREFIX_QUERIES_PER_CTA / group_size);
  int32_t nc = 0, nm = 0, max_sp = 0;
  for (int32_t first : order) {
    const auto& group = by_first[first];
    if (group.size() < 2) continue;
    const auto& lead = batch[group[0]]->pages;
    size_t common = lead.size();
    for (int32_t i : group) {
      const auto& pages = batch[i]->pages;
      size_t k = 0;
      while (k < common && k < pages.size() && pages[k] == lead[k]) ++k;
      common = k;
    }
    const int64_t shared_tokens = (int64_t)common * a->block_size;
    int64_t sp = INT64_MAX;
    for (int32_t i : group) {
      const int64_t usable = std::min(shared_tokens, batch[i]->tokens - 1);
      sp = std::min(sp, usable > 0 ? usable / PA_PARTITION_TOKENS : (int64_t)0);
    }
    if (sp <= 0) continue;
    for (size_t off = 0; off < group.size(); off += per_chunk) {
      const int32_t count = (int32_t)std::min<size_t>(per_chunk, group.size() - off);
      int32_t* c = chunks + 4 * (int64_t)nc;
      c[0] = group[0];
      c[1] = nm;
      c[2] = count;
      c[3] = (int32_t)sp;
      for (int32_t k = 0; k < count; ++k) {
        members[nm + k] = group[off + k];
        first_partition[group[off + k]] = (int32_t)sp;
      }
      nm += count;
      ++nc;
    }
    max_sp = std::max(max_sp, (int32_t)sp);
  }
  int32_t min_sp = n > 0 ? INT32_MAX : 0;
  for (int32_t i = 0; i < n; ++i) min_sp = std::min(min_sp, first_partition[i]);
  *num_chunks = nc;
  *num_members = nm;
  *max_shared_partitions = max_sp;
  *min_shared_partitions = min_sp;
  return PA_OK;
}

// Incremental export.  A row is exported whole (pad included) when its
// contents are not known to belong to the sequence's logged state: a row never
// exported, a row last exported for another sequence, a sequence last exported
// at another row, a sequence new since (allocated or forked), or one whose log
// overflowed.  Otherwise only its logged entries go out, each once, with the
// page the table holds now.  Logs are cleared and rows recorded only once the
// whole batch fits in the caller's buffer.
pa_status pa_block_alloc_table_updates(pa_block_alloc* a, const int64_t* seqs, int32_t n,
                                       int32_t max_blocks_per_seq, int32_t pad, int32_t* updates, int32_t cap,
                                       int32_t* n_out, int32_t* context_lens_out) {
  if (n_out) *n_out = 0;
  if (!a || n < 0 || max_blocks_per_seq < 0 || cap < 0 || !n_out || (n > 0 && !seqs) || (cap > 0 && !updates))
    return fail(PA_ERR_INVALID, "table_updates: bad argument");
  const bool same_width = a->rows_width == max_blocks_per_seq;
  std::vector<pa_block_alloc::Seq*> batch(n);
  std::vector<char> whole(n);
  int64_t count = 0;
  for (int32_t i = 0; i < n; ++i) {
    auto it = a->seqs.find(seqs[i]);
    if (it == a->seqs.end())
      return fail(PA_ERR_NOT_FOUND, "table_updates: unknown sequence %lld", (long long)seqs[i]);
    pa_block_alloc::Seq& sq = it->second;
    if ((int64_t)sq.pages.size() > max_blocks_per_seq)
      return fail(PA_ERR_INVALID, "table_updates: sequence %lld holds %zu pages > %d", (long long)seqs[i],
                  sq.pages.size(), max_blocks_per_seq);
    batch[i] = &sq;
    const bool known = same_width && i < (int32_t)a->row_owner.size();
    const int64_t owner = known ? a->row_owner[i] : pa_block_alloc::kNoOwner;
    whole[i] = sq.whole || sq.row != i || owner != seqs[i];
    if (whole[i]) {
      const int64_t held = owner == pa_block_alloc::kNoOwner ? max_blocks_per_seq : a->row_len[i];
      count += std::max<int64_t>((int64_t)sq.pages.size(), held);
    } else {
      std::sort(sq.changed.begin(), sq.changed.end());
      sq.changed.erase(std::unique(sq.changed.begin(), sq.changed.end()), sq.changed.end());
      count += (int64_t)sq.changed.size();
    }
  }
  *n_out = count > INT32_MAX ? INT32_MAX : (int32_t)count;
  if (count > cap)
    return fail(PA_ERR_INVALID, "table_updates: %lld updates, capacity %d", (long long)count, cap);
  if (!same_width) {
    a->row_owner.clear();
    a->row_len.clear();
    a->rows_width = max_blocks_per_seq;
  }
  if ((int32_t)a->row_owner.size() < n) {
    a->row_owner.resize(n, pa_block_alloc::kNoOwner);
    a->row_len.resize(n, 0);
  }
  int32_t* u = updates;
  auto put = [&](int32_t row, int32_t col, int32_t page) {
    u[0] = row;
    u[1] = col;
    u[2] = page;
    u += 3;
  };
  for (int32_t i = 0; i < n; ++i) {
    const pa_block_alloc::Seq& sq = *batch[i];
    const int32_t len = (int32_t)sq.pages.size();
    if (whole[i]) {
      const int32_t held =
          a->row_owner[i] == pa_block_alloc::kNoOwner ? max_blocks_per_seq : a->row_len[i];
      for (int32_t j = 0; j < len; ++j) put(i, j, sq.pages[j]);
      for (int32_t j = len; j < held; ++j) put(i, j, pad);
    } else {
      for (int32_t j : sq.changed) put(i, j, sq.pages[j]);
    }
    a->row_owner[i] = seqs[i];
    a->row_len[i] = len;
    if (context_lens_out) context_lens_out[i] = (int32_t)sq.tokens;
  }
  for (int32_t i = 0; i < n; ++i) {
    batch[i]->changed.clear();
    batch[i]->whole = false;
    batch[i]->row = i;  // a sequence at several rows: the last one
  }
  return PA_OK;
}

}  // extern "C"
