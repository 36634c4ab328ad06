// Host planner and C ABI of the masked attention forward.
//
// attn_plan() turns a problem + mask descriptor into:
//   * the class of every 128 x 128 (query, key) tile over its valid sub-rectangle
//     (empty / full / partial): empty tiles are never loaded, full tiles skip all mask
//     arithmetic, partial tiles get a 2 KiB tile-transposed bit mask (row r's 128 bits
//     at byte 16 r, bit c of the row = key c of the tile) that one thread per row reads
//     with a single 16-byte load. This replaces the per-element, uncoalesced custom-mask
//     reads that "Custom mask slows down attention." (flashinfer #724) blames for a 2x
//     slowdown, and generalises the block mask of "[Attention] feat: support PrefixLM"
//     (build_block_mask) to every kind;
//   * a work list of (query tiles, key-tile run) items, balanced over the persistent CTAs
//     of the forward by longest-processing-time-first assignment, so that ragged lengths
//     ("feat: support custom mask for flash attention": ragged paged attention) do not
//     leave SMs idle.
//
// Analytic kinds are reduced to per-row half-open key intervals on the host; range lists
// ("Feature request: chunk-causal mask type for Flex Flash Attention") are merged per row,
// so the union of many ranges classifies exactly even when no single range covers a tile.
// CUSTOM masks are scanned on the device (attn_custom.cu).
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <new>
#include <numeric>
#include <queue>
#include <unordered_map>
#include <stdexcept>
#include <utility>
#include <vector>

#include "attn_internal.h"
#include "attn_testing.h"

// 1: balance items group by group (see build_work); 0: plain longest-processing-time-first
#ifndef MFA_SCHED_GROUPED
#define MFA_SCHED_GROUPED 1
#endif

namespace {

using namespace mfa;

struct Iv {
  int32_t a, b;
};

constexpr int32_t kClassEmpty = 0, kClassFull = 1, kClassPartial = 2;

// Validated view of the problem.
struct Shape {
  int B = 0, hq = 0, hkv = 0, d = 0;
  float scale = 0.f;
  bool paged = false;
  int ps = 0, maxp = 0, npages = 0;
  std::vector<int32_t> lq, lk, qoff, koff;
  int64_t total_q = 0, total_kv_rows = 0;
  int kv_splits = 0;   // 0 automatic, 1 never, N >= 2 at most N key ranges per query tile
  int q_begin = 0, q_end = INT32_MAX;   // query-row shard (sequence-local rows)
};

attn_status_t validate_problem(const attn_problem_t* p, Shape& s, bool need_device_ptrs = true) {
  if (!p) return ATTN_ERR_INVALID_ARG;
  if (p->batch < 0 || p->hq <= 0 || p->hkv <= 0) return ATTN_ERR_INVALID_ARG;
  if (p->hq % p->hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (p->head_dim != 64 && p->head_dim != 128 && p->head_dim != 256) return ATTN_ERR_UNSUPPORTED;
  if (std::isnan(p->scale) || std::isinf(p->scale)) return ATTN_ERR_INVALID_ARG;
  if (p->kv_splits < 0) return ATTN_ERR_INVALID_ARG;
  s.kv_splits = p->kv_splits;
  if (p->q_begin < 0 || (p->q_end > 0 && p->q_end < p->q_begin)) return ATTN_ERR_INVALID_ARG;
  s.q_begin = p->q_begin;
  s.q_end = p->q_end > 0 ? p->q_end : INT32_MAX;
  s.B = p->batch;
  s.hq = p->hq;
  s.hkv = p->hkv;
  s.d = p->head_dim;
  s.scale = p->scale > 0.f ? p->scale : 1.0f / std::sqrt(float(p->head_dim));
  if (s.B > 0 && !p->cu_seqlens_q) return ATTN_ERR_INVALID_ARG;
  s.paged = p->cu_seqlens_k == nullptr;
  if (s.paged) {
    if (s.B > 0 && (!p->kv_lens || (need_device_ptrs && !p->page_table))) return ATTN_ERR_INVALID_ARG;
    if (p->page_size != 16 && p->page_size != 32 && p->page_size != 64 && p->page_size != 128)
      return ATTN_ERR_UNSUPPORTED;
    if (p->max_pages_per_seq < 0 || p->num_pages < 0) return ATTN_ERR_INVALID_ARG;
    if (int64_t(p->num_pages) * p->page_size > INT32_MAX) return ATTN_ERR_UNSUPPORTED;
    s.ps = p->page_size;
    s.maxp = p->max_pages_per_seq;
    s.npages = p->num_pages;
  } else if (p->kv_lens) {
    return ATTN_ERR_INVALID_ARG;  // both layouts given
  }
  if (s.B > 0 && p->cu_seqlens_q[0] != 0) return ATTN_ERR_INVALID_ARG;
  s.lq.resize(s.B);
  s.lk.resize(s.B);
  s.qoff.resize(s.B);
  s.koff.resize(s.B);
  for (int b = 0; b < s.B; ++b) {
    int64_t q0 = p->cu_seqlens_q[b], q1 = p->cu_seqlens_q[b + 1];
    if (q1 < q0) return ATTN_ERR_INVALID_ARG;
    s.lq[b] = int32_t(q1 - q0);
    s.qoff[b] = int32_t(q0);
    if (s.paged) {
      int64_t n = p->kv_lens[b];
      if (n < 0) return ATTN_ERR_INVALID_ARG;
      if (n > int64_t(s.maxp) * s.ps) return ATTN_ERR_INVALID_ARG;  // more keys than the page row holds
      s.lk[b] = int32_t(n);
      if (int64_t(b) * s.maxp > INT32_MAX) return ATTN_ERR_UNSUPPORTED;
      s.koff[b] = b * s.maxp;
    } else {
      if (b == 0 && p->cu_seqlens_k[0] != 0) return ATTN_ERR_INVALID_ARG;
      int64_t k0 = p->cu_seqlens_k[b], k1 = p->cu_seqlens_k[b + 1];
      if (k1 < k0) return ATTN_ERR_INVALID_ARG;
      s.lk[b] = int32_t(k1 - k0);
      s.koff[b] = int32_t(k0);
    }
  }
  s.total_q = s.B ? p->cu_seqlens_q[s.B] : 0;
  s.total_kv_rows = s.paged ? int64_t(s.npages) * s.ps : (s.B ? p->cu_seqlens_k[s.B] : 0);
  return ATTN_OK;
}

bool range_ok(const attn_range_t& r) {
  if (r.q_start < 0 || r.q_end < r.q_start || r.k_start < 0 || r.k_end < r.k_start) return false;
  if (r.type != ATTN_RANGE_FULL && r.type != ATTN_RANGE_CAUSAL && r.type != ATTN_RANGE_INV_CAUSAL &&
      r.type != ATTN_RANGE_BI_CAUSAL && r.type != ATTN_RANGE_CHUNK_CAUSAL)
    return false;
  if (r.type == ATTN_RANGE_CHUNK_CAUSAL && r.chunk_size < 1) return false;
  return true;
}

attn_status_t validate_mask(const attn_mask_desc_t* m, const Shape& s) {
  if (!m) return ATTN_ERR_INVALID_ARG;
  switch (m->kind) {
    case ATTN_MASK_FULL:
    case ATTN_MASK_CAUSAL:
      return ATTN_OK;
    case ATTN_MASK_SLIDING_WINDOW:
      return m->window >= 1 ? ATTN_OK : ATTN_ERR_INVALID_ARG;
    case ATTN_MASK_PREFIX_LM:
      if (m->prefix_lens) {
        for (int b = 0; b < s.B; ++b)
          if (m->prefix_lens[b] < 0) return ATTN_ERR_INVALID_ARG;
        return ATTN_OK;
      }
      return m->prefix_len >= 0 ? ATTN_OK : ATTN_ERR_INVALID_ARG;
    case ATTN_MASK_CHUNK_CAUSAL:
      if (m->chunk.type != ATTN_RANGE_CHUNK_CAUSAL || !range_ok(m->chunk)) return ATTN_ERR_INVALID_ARG;
      return ATTN_OK;
    case ATTN_MASK_RANGES: {
      if (s.B > 0 && (!m->cu_ranges || m->cu_ranges[0] != 0)) return ATTN_ERR_INVALID_ARG;
      for (int b = 0; b < s.B; ++b) {
        if (m->cu_ranges[b + 1] < m->cu_ranges[b]) return ATTN_ERR_INVALID_ARG;
        if (m->cu_ranges[b + 1] > m->cu_ranges[b] && !m->ranges) return ATTN_ERR_INVALID_ARG;
        for (int32_t r = m->cu_ranges[b]; r < m->cu_ranges[b + 1]; ++r) {
          const attn_range_t& g = m->ranges[r];
          if (!range_ok(g) || g.q_end > s.lq[b] || g.k_end > s.lk[b]) return ATTN_ERR_INVALID_ARG;
        }
      }
      return ATTN_OK;
    }
    case ATTN_MASK_BLOCK_SPARSE: {
      if (m->block_q < 1 || m->block_k < 1) return ATTN_ERR_INVALID_ARG;
      if (s.B == 0) return ATTN_OK;
      if (!m->bsr_row_ptr || m->bsr_row_ptr[0] != 0) return ATTN_ERR_INVALID_ARG;
      int64_t row = 0;
      for (int b = 0; b < s.B; ++b) {
        const int64_t nbr = (int64_t(s.lq[b]) + m->block_q - 1) / m->block_q;
        const int64_t nbc = (int64_t(s.lk[b]) + m->block_k - 1) / m->block_k;
        for (int64_t r = row; r < row + nbr; ++r) {
          if (m->bsr_row_ptr[r + 1] < m->bsr_row_ptr[r]) return ATTN_ERR_INVALID_ARG;
          if (m->bsr_row_ptr[r + 1] > m->bsr_row_ptr[r] && !m->bsr_col_idx) return ATTN_ERR_INVALID_ARG;
          for (int32_t e = m->bsr_row_ptr[r]; e < m->bsr_row_ptr[r + 1]; ++e)
            if (m->bsr_col_idx[e] < 0 || m->bsr_col_idx[e] >= nbc) return ATTN_ERR_INVALID_ARG;
        }
        row += nbr;
      }
      return ATTN_OK;
    }
    case ATTN_MASK_CUSTOM: {
      if (s.B == 0) return ATTN_OK;
      if (!m->mask_word_offsets) return ATTN_ERR_INVALID_ARG;
      if (m->mask_words_total < 0) return ATTN_ERR_INVALID_ARG;
      int64_t need_end = 0;
      for (int b = 0; b < s.B; ++b) {
        int64_t o0 = m->mask_word_offsets[b], o1 = m->mask_word_offsets[b + 1];
        if (o0 < 0 || o1 < o0) return ATTN_ERR_INVALID_ARG;
        int64_t need = int64_t(s.lq[b]) * ((int64_t(s.lk[b]) + 31) / 32);
        // "custom_mask length must be larger than total kv length" (sglang-jax PR #20 review)
        if (o1 - o0 < need) return ATTN_ERR_MASK_TOO_SMALL;
        need_end = std::max(need_end, o0 + need);
      }
      if (need_end > m->mask_words_total) return ATTN_ERR_MASK_TOO_SMALL;
      if (need_end > 0 && !m->mask_bits) return ATTN_ERR_INVALID_ARG;
      return ATTN_OK;
    }
    default:
      return ATTN_ERR_INVALID_ARG;
  }
}

// Per-row key intervals of the analytic kinds (everything but CUSTOM).
class RowSource {
 public:
  RowSource(const attn_mask_desc_t* m, const Shape& s) : m_(m), s_(s) {}

  // Build the merged per-row intervals of sequence b for the range and block-sparse kinds.
  void prepare(int b) {
    if (m_->kind == ATTN_MASK_BLOCK_SPARSE) return prepare_bsr(b);
    if (m_->kind != ATTN_MASK_RANGES && m_->kind != ATTN_MASK_CHUNK_CAUSAL) return;
    const int lq = s_.lq[b], lk = s_.lk[b];
    std::vector<attn_range_t> rs;
    if (m_->kind == ATTN_MASK_RANGES) {
      for (int32_t r = m_->cu_ranges[b]; r < m_->cu_ranges[b + 1]; ++r) rs.push_back(m_->ranges[r]);
    } else {
      const attn_range_t& c = m_->chunk;
      rs.push_back(attn_range_t{0, c.q_start, 0, c.q_start, ATTN_RANGE_CAUSAL, 0});
      rs.push_back(c);
    }
    off_.assign(size_t(lq) + 1, 0);
    for (const auto& r : rs) {
      int32_t a = std::min(r.q_start, lq), e = std::min(r.q_end, lq);
      for (int32_t i = a; i < e; ++i) off_[i + 1]++;
    }
    for (int i = 0; i < lq; ++i) off_[i + 1] += off_[i];
    iv_.assign(off_[lq], Iv{0, 0});
    std::vector<int64_t> fill(off_.begin(), off_.end() - 1);
    for (const auto& r : rs) {
      int32_t a = std::min(r.q_start, lq), e = std::min(r.q_end, lq);
      for (int32_t i = a; i < e; ++i) {
        int64_t lo = std::max<int64_t>(r.k_start, 0), hi = std::min<int64_t>(r.k_end, lk);
        if (r.type == ATTN_RANGE_CAUSAL) {
          hi = std::min<int64_t>(hi, int64_t(i) + 1);
        } else if (r.type == ATTN_RANGE_INV_CAUSAL || r.type == ATTN_RANGE_BI_CAUSAL) {
          lo = std::max<int64_t>(lo, int64_t(r.k_start) + (int64_t(i) - r.q_start));
          if (r.type == ATTN_RANGE_BI_CAUSAL)
            hi = std::min<int64_t>(hi, int64_t(r.k_end) - (int64_t(r.q_end) - i) + 1);
        } else if (r.type == ATTN_RANGE_CHUNK_CAUSAL) {
          int64_t c = (int64_t(i) - r.q_start) / r.chunk_size;
          int64_t end = std::min<int64_t>(int64_t(r.q_start) + (c + 1) * int64_t(r.chunk_size), r.q_end);
          hi = std::min(hi, end);
        }
        iv_[fill[i]++] = lo < hi ? Iv{int32_t(lo), int32_t(hi)} : Iv{0, 0};
      }
    }
    // merge each row in place (sort by start; drop empties; coalesce overlaps/adjacency)
    std::vector<int64_t> noff(size_t(lq) + 1, 0);
    int64_t w = 0;
    for (int i = 0; i < lq; ++i) {
      auto first = iv_.begin() + off_[i], last = iv_.begin() + off_[i + 1];
      std::sort(first, last, [](const Iv& x, const Iv& y) { return x.a < y.a; });
      int64_t row_start = w;
      for (auto it = first; it != last; ++it) {
        if (it->a >= it->b) continue;
        if (w > row_start && it->a <= iv_[w - 1].b) {
          iv_[w - 1].b = std::max(iv_[w - 1].b, it->b);
        } else {
          iv_[w++] = *it;
        }
      }
      noff[i + 1] = w;
    }
    iv_.resize(w);
    off_.swap(noff);
  }

  // Block-sparse: every row of block row R shares the intervals of R's listed block columns.
  void prepare_bsr(int b) {
    const int lq = s_.lq[b], lk = s_.lk[b], bq = m_->block_q, bk = m_->block_k;
    int64_t row0 = 0;
    for (int x = 0; x < b; ++x) row0 += (int64_t(s_.lq[x]) + bq - 1) / bq;
    const int nbr = (lq + bq - 1) / bq;
    std::vector<Iv> brow;
    off_.assign(size_t(lq) + 1, 0);
    iv_.clear();
    for (int R = 0; R < nbr; ++R) {
      brow.clear();
      for (int32_t e = m_->bsr_row_ptr[row0 + R]; e < m_->bsr_row_ptr[row0 + R + 1]; ++e) {
        const int64_t a = int64_t(m_->bsr_col_idx[e]) * bk;
        brow.push_back(Iv{int32_t(a), int32_t(std::min<int64_t>(a + bk, lk))});
      }
      std::sort(brow.begin(), brow.end(), [](const Iv& x, const Iv& y) { return x.a < y.a; });
      std::vector<Iv> merged;
      for (const Iv& v : brow) {
        if (v.a >= v.b) continue;
        if (!merged.empty() && v.a <= merged.back().b) merged.back().b = std::max(merged.back().b, v.b);
        else merged.push_back(v);
      }
      const int r_end = std::min(lq, (R + 1) * bq);
      for (int i = R * bq; i < r_end; ++i) {
        iv_.insert(iv_.end(), merged.begin(), merged.end());
        off_[i + 1] = int64_t(iv_.size());
      }
    }
  }

  // Intervals of row i of sequence b (sorted, disjoint, non-empty, inside [0, L_k)).
  int row(int b, int i, const Iv** out) {
    const int64_t lq = s_.lq[b], lk = s_.lk[b];
    const int64_t pos = int64_t(i) + lk - lq;
    int n = 0;
    auto emit = [&](int64_t a, int64_t e) {
      a = std::max<int64_t>(a, 0);
      e = std::min<int64_t>(e, lk);
      if (a < e) buf_[n++] = Iv{int32_t(a), int32_t(e)};
    };
    switch (m_->kind) {
      case ATTN_MASK_FULL:
        emit(0, lk);
        break;
      case ATTN_MASK_CAUSAL:
        emit(0, pos + 1);
        break;
      case ATTN_MASK_SLIDING_WINDOW:
        emit(pos - int64_t(m_->window) + 1, pos + 1);
        break;
      case ATTN_MASK_PREFIX_LM: {
        int64_t p = m_->prefix_lens ? m_->prefix_lens[b] : m_->prefix_len;
        emit(0, std::max(p, pos + 1));
        break;
      }
      default:
        *out = iv_.data() + off_[i];
        return int(off_[i + 1] - off_[i]);
    }
    *out = buf_;
    return n;
  }

 private:
  const attn_mask_desc_t* m_;
  const Shape& s_;
  std::vector<int64_t> off_;
  std::vector<Iv> iv_;
  Iv buf_[2];
};

// Visible-pair counts of every (row block of R rows, key tile) of one sequence.
void count_sequence(RowSource& src, int b, const Shape& s, int R, std::vector<int32_t>& cnt) {
  const int lq = s.lq[b], lk = s.lk[b];
  const int n_rb = (lq + R - 1) / R, n_kt = (lk + kTile - 1) / kTile;
  cnt.assign(size_t(n_rb) * n_kt, 0);
  std::vector<int32_t> diff(size_t(n_kt) + 1);
  for (int rb = 0; rb < n_rb; ++rb) {
    int32_t* c = cnt.data() + size_t(rb) * n_kt;
    std::fill(diff.begin(), diff.end(), 0);
    const int r_end = std::min(lq, (rb + 1) * R);
    for (int i = rb * R; i < r_end; ++i) {
      const Iv* iv;
      int n = src.row(b, i, &iv);
      for (int t = 0; t < n; ++t) {
        const int a = iv[t].a, e = iv[t].b;
        const int ka = a / kTile, kb = (e - 1) / kTile;
        if (ka == kb) {
          c[ka] += e - a;
        } else {
          c[ka] += (ka + 1) * kTile - a;
          c[kb] += e - kb * kTile;
          diff[ka + 1] += 1;
          diff[kb] -= 1;
        }
      }
    }
    int32_t run = 0;
    for (int kt = 0; kt < n_kt; ++kt) {
      run += diff[kt];
      c[kt] += run * kTile;
    }
  }
}

inline int32_t classify(int64_t cnt, int64_t total) {
  return cnt == 0 ? kClassEmpty : (cnt == total ? kClassFull : kClassPartial);
}

// 128 x 128 classes of one sequence from its R-row block counts.
void report_classes(const std::vector<int32_t>& cnt, int lq, int lk, int R, std::vector<uint8_t>& out,
                    attn_plan_stats_t& st) {
  const int n_rb = (lq + R - 1) / R, n_kt = (lk + kTile - 1) / kTile;
  const int n_qt = (lq + kTile - 1) / kTile, per = kTile / R;
  for (int qt = 0; qt < n_qt; ++qt) {
    const int64_t rows = std::min(kTile, lq - qt * kTile);
    for (int kt = 0; kt < n_kt; ++kt) {
      int64_t c = 0;
      for (int rb = qt * per; rb < std::min(n_rb, (qt + 1) * per); ++rb) c += cnt[size_t(rb) * n_kt + kt];
      const int64_t cols = std::min(kTile, lk - kt * kTile);
      const int32_t k = classify(c, rows * cols);
      out.push_back(uint8_t(k));
      st.unmasked_pairs += c;
      if (k == kClassEmpty) st.tiles_empty++;
      else if (k == kClassFull) st.tiles_full++;
      else st.tiles_partial++;
    }
  }
}

struct TileRef {
  int32_t seq, rb, kt, idx;
};

// Work list for all sequences given their R-row block counts.
struct WorkList {
  std::vector<WorkItem> items;
  std::vector<Job> jobs;
  std::vector<TileRef> mask_tiles;   // in index order
  std::vector<int32_t> cta_off, cta_items;
  std::vector<MergeTile> merge;      // split-KV: query tiles to merge
  int32_t slots = 0;                 // split-KV: partial-result slots
  int32_t splits_max = 1;
};

// Greedy least-loaded assignment of costs (taken in the given order) onto `units`: the
// largest load, i.e. the modelled makespan.
int64_t greedy_makespan(const std::vector<int64_t>& costs, int units) {
  using Load = std::pair<int64_t, int32_t>;
  std::priority_queue<Load, std::vector<Load>, std::greater<Load>> heap;
  for (int c = 0; c < units; ++c) heap.push(Load{0, c});
  int64_t worst = 0;
  for (int64_t x : costs) {
    Load l = heap.top();
    heap.pop();
    l.first += x;
    worst = std::max(worst, l.first);
    heap.push(l);
  }
  return worst;
}

// Split-KV. A work item's key tiles may be cut into n consecutive ranges, each a work item
// of its own that writes partial results (out / l and lse per row) to its own slots; the
// merge kernel combines them by lse. Forced (kv_splits = N >= 2): every item with >= 2 key
// tiles into min(N, tiles) ranges. Automatic (kv_splits = 0): a cost model in key-tile
// units -- an item (or range) costs its tiles + 2 (Q load, pipeline start, epilogue), the
// merge costs one tile per partial slot spread over all units -- picks the range length
// P = ceil(longest / n), n = 1 .. 64, whose longest-first greedy schedule plus merge is
// shortest; the split is kept only when that beats the unsplit makespan by more than 15 %.
void split_items(const Shape& s, int units, int nq, WorkList& wl) {
  if (s.kv_splits == 1 || wl.items.empty()) return;
  auto pieces_of = [&](const WorkItem& it, int64_t P) -> int {
    int n = 1;
    if (s.kv_splits >= 2) n = it.job_count >= 2 ? std::min(s.kv_splits, it.job_count) : 1;
    else if (P > 0) n = int((it.job_count + P - 1) / P);
    return std::max(1, std::min(n, kMaxSplits));
  };
  int64_t best_P = 0;   // 0: no split
  if (s.kv_splits == 0) {
    int64_t longest = 0;
    for (const WorkItem& it : wl.items) longest = std::max<int64_t>(longest, it.job_count);
    auto cost = [&](int64_t P) {
      std::vector<int64_t> costs;
      int64_t slots = 0;
      for (const WorkItem& it : wl.items) {
        const int n = P > 0 ? pieces_of(it, P) : 1;
        for (int c = 0; c < n; ++c)
          costs.push_back(int64_t(it.job_count) * (c + 1) / n - int64_t(it.job_count) * c / n + 2);
        if (n > 1) slots += int64_t(n) * nq;
      }
      std::sort(costs.begin(), costs.end(), std::greater<int64_t>());
      return greedy_makespan(costs, units) + (slots + units - 1) / units;
    };
    const int64_t base = cost(0);
    int64_t total = 0;
    for (const WorkItem& it : wl.items) total += it.job_count + 2;
    if (100 * base <= 115 * ((total + units - 1) / units)) return;   // already balanced
    int64_t best = base;
    for (int n = 2; n <= 64; ++n) {
      const int64_t P = std::max<int64_t>(4, (longest + n - 1) / n);
      const int64_t c = cost(P);
      if (c < best) {
        best = c;
        best_P = P;
      }
      if (P == 4) break;
    }
    if (best_P == 0 || 100 * best >= 85 * base) return;
  }
  std::vector<WorkItem> out;
  out.reserve(wl.items.size());
  for (const WorkItem& it : wl.items) {
    const int n = pieces_of(it, best_P);
    if (n <= 1) {
      out.push_back(it);
      continue;
    }
    const int32_t slot0 = wl.slots;
    for (int c = 0; c < n; ++c) {
      WorkItem p = it;
      const int32_t j0 = int32_t(int64_t(it.job_count) * c / n), j1 = int32_t(int64_t(it.job_count) * (c + 1) / n);
      p.job_start = it.job_start + j0;
      p.job_count = j1 - j0;
      p.part = slot0 + c * nq;
      out.push_back(p);
    }
    wl.slots += n * nq;
    for (int t = 0; t < nq; ++t)
      if (it.rows[t] > 0) wl.merge.push_back(MergeTile{it.tok[t], it.head[t], it.rows[t], slot0 + t, n, nq, {0, 0}});
    wl.splits_max = std::max(wl.splits_max, n);
  }
  wl.items.swap(out);
}

// Column of sequence b in a transposed V whose sequences start at multiples of 128 keys
// (the e4m3 forward's TMA needs 16-byte aligned starts): offsets[B + 1].
std::vector<int32_t> vt_offsets(const Shape& s) {
  std::vector<int32_t> off(size_t(s.B) + 1, 0);
  for (int b = 0; b < s.B; ++b) off[b + 1] = off[b] + (s.lk[b] + kTile - 1) / kTile * kTile;
  return off;
}

void build_work(const Shape& s, int R, int hp, int nq, const std::vector<std::vector<int32_t>>& cnts,
                int num_sms, WorkList& wl, bool allow_split = true) {
  const int g = s.hq / s.hkv;
  const int G = g / hp;  // head groups per kv head
  const std::vector<int32_t> vt_off = vt_offsets(s);
  for (int b = 0; b < s.B; ++b) {
    const int lq = s.lq[b], lk = s.lk[b];
    if (lq == 0) continue;
    const int n_rb = (lq + R - 1) / R, n_kt = (lk + kTile - 1) / kTile;
    const std::vector<int32_t>& cnt = cnts[b];
    std::vector<int32_t> tidx(size_t(n_rb) * n_kt, -1);
    std::unordered_map<int64_t, std::pair<int32_t, int32_t>> lists;   // (row blocks) -> jobs
    auto kclass = [&](int rb, int kt) -> int32_t {
      const int64_t rows = std::min(R, lq - rb * R), cols = std::min(kTile, lk - kt * kTile);
      return classify(cnt[size_t(rb) * n_kt + kt], rows * cols);
    };
    auto mask_of = [&](int rb, int kt) -> int32_t {
      if (rb < 0) return kMaskNone;
      const int32_t k = kclass(rb, kt);
      if (k == kClassEmpty) return kMaskNone;
      // a full tile that extends past L_k still needs its key columns cut
      if (k == kClassFull && (kt + 1) * kTile <= lk) return kMaskFull;
      int32_t& t = tidx[size_t(rb) * n_kt + kt];
      if (t < 0) {
        t = int32_t(wl.mask_tiles.size());
        wl.mask_tiles.push_back(TileRef{b, rb, kt, t});
      }
      return t;
    };
    auto add_item = [&](int kh, int rb0, int hg0, int rb1, int hg1) {
      WorkItem it{};
      it.part = -1;
      it.vt_base = s.paged ? 0 : vt_off[b];
      it.seq = b;
      it.kv_head = kh;
      it.k_base = s.koff[b];
      it.kv_len = lk;
      it.npages = s.paged ? (lk + s.ps - 1) / s.ps : 0;
      const int rbs[2] = {rb0, rb1}, hgs[2] = {hg0, hg1};
      for (int t = 0; t < 2; ++t) {
        const int rb = rbs[t] >= 0 ? rbs[t] : rb0, hg = rbs[t] >= 0 ? hgs[t] : hg0;
        it.tok[t] = s.qoff[b] + rb * R;
        it.rows[t] = rbs[t] >= 0 ? std::min(R, lq - rb * R) : 0;
        it.head[t] = kh * g + hg * hp;
      }
      // The jobs depend on the row blocks only, not on the heads: items of other KV heads
      // and head groups over the same row blocks share one list (read-only on the device).
      const int64_t key = int64_t(rb0) * (int64_t(n_rb) + 1) + (rb1 + 1);
      auto hit = lists.find(key);
      if (hit != lists.end()) {
        it.job_start = hit->second.first;
        it.job_count = hit->second.second;
        wl.items.push_back(it);
        return;
      }
      it.job_start = int32_t(wl.jobs.size());
      for (int kt = 0; kt < n_kt; ++kt) {
        Job j{};
        j.k_tile = kt;
        j.mask[0] = mask_of(rb0, kt);
        j.mask[1] = nq == 2 ? mask_of(rb1, kt) : kMaskNone;
        if (j.mask[0] == kMaskNone && j.mask[1] == kMaskNone) continue;
        wl.jobs.push_back(j);
      }
      if (wl.jobs.size() == size_t(it.job_start)) {
        // every row of the item is fully masked: one hidden job writes out = 0, lse = -inf
        wl.jobs.push_back(Job{0, {kMaskNone, kMaskNone}, 0});
      }
      it.job_count = int32_t(wl.jobs.size()) - it.job_start;
      lists.emplace(key, std::make_pair(it.job_start, it.job_count));
      wl.items.push_back(it);
    };
    // the row blocks this plan computes: those overlapping the query-row shard
    const int rb0 = std::min(n_rb, s.q_begin / R);
    const int rb1 = std::min<int64_t>(n_rb, (std::min<int64_t>(s.q_end, lq) + R - 1) / R);
    for (int kh = 0; kh < s.hkv; ++kh) {
      if (nq == 2 && G >= 2) {
        for (int rb = rb0; rb < rb1; ++rb)
          for (int hg = 0; hg < G; hg += 2) add_item(kh, rb, hg, hg + 1 < G ? rb : -1, hg + 1);
      } else if (nq == 2) {
        for (int rb = rb0; rb < rb1; rb += 2) add_item(kh, rb, 0, rb + 1 < rb1 ? rb + 1 : -1, 0);
      } else {
        for (int rb = rb0; rb < rb1; ++rb)
          for (int hg = 0; hg < G; ++hg) add_item(kh, rb, hg, -1, 0);
      }
    }
  }
  if (allow_split) split_items(s, num_sms, nq, wl);
  // Greedy balancing onto persistent CTAs: each item goes to the least-loaded CTA. Items are
  // taken group by group -- a group being one (sequence, key/value head), the largest
  // groups first -- and, inside a group, longest first. Items of one group then run at
  // about the same time on different CTAs and share their K/V tiles in L2 (pure
  // longest-first interleaves every group and re-reads K/V from DRAM once it exceeds L2);
  // with one item per group this is plain longest-processing-time-first.
  const int n_items = int(wl.items.size());
  const int C = std::max(1, std::min(num_sms, n_items));
  std::vector<int32_t> order(n_items);
  std::iota(order.begin(), order.end(), 0);
  auto group = [&](int32_t i) { return int64_t(wl.items[i].seq) * s.hkv + wl.items[i].kv_head; };
  std::vector<int64_t> gcost(size_t(s.B) * s.hkv, 0);
  for (const WorkItem& it : wl.items) gcost[size_t(it.seq) * s.hkv + it.kv_head] += it.job_count;
  std::stable_sort(order.begin(), order.end(), [&](int32_t x, int32_t y) {
    if (MFA_SCHED_GROUPED && group(x) != group(y)) {
      const int64_t cx = gcost[group(x)], cy = gcost[group(y)];
      return cx != cy ? cx > cy : group(x) < group(y);
    }
    return wl.items[x].job_count > wl.items[y].job_count;
  });
  using Load = std::pair<int64_t, int32_t>;
  std::priority_queue<Load, std::vector<Load>, std::greater<Load>> heap;
  for (int c = 0; c < C; ++c) heap.push(Load{0, c});
  std::vector<std::vector<int32_t>> per(C);
  for (int32_t it : order) {
    Load l = heap.top();
    heap.pop();
    per[l.second].push_back(it);
    l.first += int64_t(wl.items[it].job_count) + 1;
    heap.push(l);
  }
  wl.cta_off.assign(size_t(C) + 1, 0);
  wl.cta_items.clear();
  for (int c = 0; c < C; ++c) {
    wl.cta_items.insert(wl.cta_items.end(), per[c].begin(), per[c].end());
    wl.cta_off[c + 1] = int32_t(wl.cta_items.size());
  }
}

// Tile-transposed bits of one mask tile from the row intervals.
void write_mask_tile(RowSource& src, const Shape& s, int R, const TileRef& t, uint32_t* dst) {
  std::memset(dst, 0, kMaskTileBytes);
  const int lq = s.lq[t.seq], lk = s.lk[t.seq];
  const int c0 = t.kt * kTile, c1 = std::min(lk, c0 + kTile);
  for (int lr = 0; lr < R; ++lr) {
    const int i = t.rb * R + lr;
    if (i >= lq) break;
    uint32_t w[4] = {0, 0, 0, 0};
    const Iv* iv;
    const int n = src.row(t.seq, i, &iv);
    for (int k = 0; k < n; ++k) {
      // bits [lo, hi) of the tile row, a word at a time
      const int lo = std::max(iv[k].a, c0) - c0, hi = std::min(iv[k].b, c1) - c0;
      for (int x = lo; x < hi;) {
        const int word = x >> 5, end = std::min(hi, (word + 1) * 32), len = end - x;
        w[word] |= (len == 32 ? ~0u : ((1u << len) - 1u)) << (x & 31);
        x = end;
      }
    }
    for (int r = lr; r < kTile; r += R) std::memcpy(dst + 4 * r, w, 16);
  }
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct Staging {
  size_t off_items, off_jobs, off_cta_off, off_cta_items, off_seq, off_tiles, off_merge, off_part_lse, off_part_o,
      total;
};

// [status | items | jobs | cta_off | cta_items | cu_k, vt_off | mask tiles | merge tiles |
//  partial lse | partial out]
Staging layout(const WorkList& wl, int d, int batch) {
  Staging st{};
  st.off_items = 256;
  st.off_jobs = align256(st.off_items + wl.items.size() * sizeof(WorkItem));
  st.off_cta_off = align256(st.off_jobs + wl.jobs.size() * sizeof(Job));
  st.off_cta_items = align256(st.off_cta_off + wl.cta_off.size() * sizeof(int32_t));
  st.off_seq = align256(st.off_cta_items + wl.cta_items.size() * sizeof(int32_t));
  st.off_tiles = align256(st.off_seq + 2 * (size_t(batch) + 1) * sizeof(int32_t));
  st.off_merge = align256(st.off_tiles + wl.mask_tiles.size() * size_t(kMaskTileBytes));
  st.off_part_lse = align256(st.off_merge + wl.merge.size() * sizeof(MergeTile));
  st.off_part_o = align256(st.off_part_lse + size_t(wl.slots) * kSlotRows * sizeof(float));
  st.total = st.off_part_o + size_t(wl.slots) * kSlotRows * size_t(d) * sizeof(float);
  return st;
}

// Kernel shape: every work item holds two 128-row query tiles; head_dim 256 runs them on a
// pair of SMs (one tile per CTA, 2-SM MMAs: each SM streams half of K and V), head_dim 64
// and 128 on one SM (two softmax warpgroups share its exponential unit better; measured).
void choose_shape(const Shape& s, attn_plan_t& m);

int choose_hp(const Shape& s) {
  const int g = s.hq / s.hkv;
  int lmax = 0;
  for (int b = 0; b < s.B; ++b) lmax = std::max(lmax, s.lq[b]);
  int hp = 1;
  while (hp * 2 <= g && g % (hp * 2) == 0 && kTile / (hp * 2) >= std::max(lmax, 8)) hp *= 2;
  return hp;
}

void choose_shape(const Shape& s, attn_plan_t& m) {
  m.nq = 2;
  m.cluster = s.d == 256 ? 2 : 1;
  m.hp = choose_hp(s);
  m.R = kTile / m.hp;
}

attn_status_t cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return ATTN_OK;
  if (e == cudaErrorMemoryAllocation) return ATTN_ERR_OOM;
  return ATTN_ERR_CUDA;
}

// CUSTOM: counts of every (row block, key tile) from the packed bits on the device.
attn_status_t custom_counts(const attn_mask_desc_t* m, const Shape& s, int R, cudaStream_t stream,
                            std::vector<std::vector<int32_t>>& cnts) {
  std::vector<CustomSeq> seqs(s.B);
  std::vector<CountTask> tasks;
  int64_t total = 0;
  for (int b = 0; b < s.B; ++b) {
    CustomSeq& c = seqs[b];
    c.word_off = m->mask_word_offsets[b];
    c.lq = s.lq[b];
    c.lk = s.lk[b];
    c.n_rb = (c.lq + R - 1) / R;
    c.n_kt = (c.lk + kTile - 1) / kTile;
    c.cnt_off = total;
    total += int64_t(c.n_rb) * c.n_kt;
    for (int rb = 0; rb < c.n_rb; ++rb)
      for (int kt = 0; kt < c.n_kt; kt += 32) tasks.push_back(CountTask{b, rb, kt, 0});
  }
  for (int b = 0; b < s.B; ++b) cnts[b].assign(size_t(seqs[b].n_rb) * seqs[b].n_kt, 0);
  if (tasks.empty()) return ATTN_OK;
  void* tmp = nullptr;
  const size_t bytes_seqs = align256(seqs.size() * sizeof(CustomSeq));
  const size_t bytes_tasks = align256(tasks.size() * sizeof(CountTask));
  const size_t bytes = bytes_seqs + bytes_tasks + size_t(total) * sizeof(int32_t);
  cudaError_t e = cudaMalloc(&tmp, bytes);
  if (e != cudaSuccess) return cuda_status(e);
  auto* d_seqs = reinterpret_cast<CustomSeq*>(tmp);
  auto* d_tasks = reinterpret_cast<CountTask*>(static_cast<char*>(tmp) + bytes_seqs);
  auto* d_cnt = reinterpret_cast<int32_t*>(static_cast<char*>(tmp) + bytes_seqs + bytes_tasks);
  std::vector<int32_t> host(total);
  e = cudaMemcpyAsync(d_seqs, seqs.data(), seqs.size() * sizeof(CustomSeq), cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(d_tasks, tasks.data(), tasks.size() * sizeof(CountTask), cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(d_cnt, 0, size_t(total) * sizeof(int32_t), stream);
  if (e == cudaSuccess) e = launch_custom_count(m->mask_bits, d_seqs, d_tasks, int(tasks.size()), R, d_cnt, stream);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(host.data(), d_cnt, size_t(total) * sizeof(int32_t), cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  cudaFree(tmp);
  if (e != cudaSuccess) return cuda_status(e);
  for (int b = 0; b < s.B; ++b)
    std::copy(host.begin() + seqs[b].cnt_off, host.begin() + seqs[b].cnt_off + cnts[b].size(), cnts[b].begin());
  return ATTN_OK;
}

attn_status_t custom_repack(const attn_mask_desc_t* m, const Shape& s, int R, const std::vector<TileRef>& mask_tiles,
                            uint4* d_tiles, cudaStream_t stream) {
  if (mask_tiles.empty()) return ATTN_OK;
  std::vector<CustomSeq> seqs(s.B);
  for (int b = 0; b < s.B; ++b) {
    seqs[b].word_off = m->mask_word_offsets[b];
    seqs[b].lq = s.lq[b];
    seqs[b].lk = s.lk[b];
    seqs[b].n_rb = (s.lq[b] + R - 1) / R;
    seqs[b].n_kt = (s.lk[b] + kTile - 1) / kTile;
  }
  std::vector<RepackTask> tasks(mask_tiles.size());
  for (size_t i = 0; i < tasks.size(); ++i) {
    const TileRef& t = mask_tiles[i];
    tasks[i] = RepackTask{t.seq, t.rb, t.kt, t.idx};
  }
  void* tmp = nullptr;
  const size_t bytes_seqs = align256(seqs.size() * sizeof(CustomSeq));
  cudaError_t e = cudaMalloc(&tmp, bytes_seqs + tasks.size() * sizeof(RepackTask));
  if (e != cudaSuccess) return cuda_status(e);
  auto* d_seqs = reinterpret_cast<CustomSeq*>(tmp);
  auto* d_tasks = reinterpret_cast<RepackTask*>(static_cast<char*>(tmp) + bytes_seqs);
  e = cudaMemcpyAsync(d_seqs, seqs.data(), seqs.size() * sizeof(CustomSeq), cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(d_tasks, tasks.data(), tasks.size() * sizeof(RepackTask), cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess)
    e = launch_custom_repack(m->mask_bits, d_seqs, d_tasks, int(tasks.size()), R, d_tiles, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  cudaFree(tmp);
  return cuda_status(e);
}

// Work-list part of the plan statistics.
void work_stats(const attn_plan_t& m, const WorkList& wl, attn_plan_stats_t& st) {
  st.mask_tiles = int64_t(wl.mask_tiles.size());
  st.work_items = int64_t(wl.items.size());
  int64_t jobs = 0;
  for (const WorkItem& it : wl.items) jobs += it.job_count;   // a split item's ranges share its jobs
  st.jobs = jobs;
  st.mask_tile_reads = 0;
  for (const WorkItem& it : wl.items)
    for (int j = it.job_start; j < it.job_start + it.job_count; ++j)
      for (int t = 0; t < 2; ++t) st.mask_tile_reads += wl.jobs[j].mask[t] >= 0 ? 1 : 0;
  st.ctas = m.ctas * m.cluster;
  st.heads_per_tile = m.hp;
  st.tiles_per_cta = m.nq / m.cluster;
  st.cluster_size = m.cluster;
  st.kv_splits_max = wl.splits_max;
  st.merge_tiles = int32_t(wl.merge.size());
  st.vt_keys = m.vt_keys;
}

// ---- backward planning ----------------------------------------------------------------

// Greedy least-loaded assignment of items (costs) onto units, group by group: groups (items
// sharing the tiles they stream, i.e. one (sequence, key/value head)) go out largest first and
// their items longest first, so that the units working on one group at a time find its
// tiles in L2. Returns per-unit offsets and item lists.
void assign_lpt(const std::vector<int64_t>& cost, const std::vector<int64_t>& group, int units,
                std::vector<int32_t>& off, std::vector<int32_t>& list) {
  const int n = int(cost.size());
  const int C = std::max(1, std::min(units, n));
  std::vector<int32_t> order(n);
  std::iota(order.begin(), order.end(), 0);
  std::unordered_map<int64_t, int64_t> gcost;
  for (int i = 0; i < n; ++i) gcost[group[i]] += cost[i];
  std::stable_sort(order.begin(), order.end(), [&](int32_t x, int32_t y) {
    if (group[x] != group[y]) {
      const int64_t cx = gcost[group[x]], cy = gcost[group[y]];
      return cx != cy ? cx > cy : group[x] < group[y];
    }
    return cost[x] > cost[y];
  });
  using Load = std::pair<int64_t, int32_t>;
  std::priority_queue<Load, std::vector<Load>, std::greater<Load>> heap;
  for (int c = 0; c < C; ++c) heap.push(Load{0, c});
  std::vector<std::vector<int32_t>> per(C);
  for (int32_t it : order) {
    Load l = heap.top();
    heap.pop();
    per[l.second].push_back(it);
    l.first += cost[it];
    heap.push(l);
  }
  off.assign(size_t(C) + 1, 0);
  list.clear();
  for (int c = 0; c < C; ++c) {
    list.insert(list.end(), per[c].begin(), per[c].end());
    off[c + 1] = int32_t(list.size());
  }
}

// Backward lists over 128-row tiles of one head (cnts: per sequence, (query tile, key tile)
// visible-pair counts with R = 128). A tile gets a mask tile when it is partial, or full but
// cut by the end of the keys or of the queries (the dK/dV kernel must not let the rows past
// L_q, which belong to the next sequence, into its sums).
struct BwdLists {
  std::vector<BwdItem> q_items, kv_items;
  std::vector<BwdJob> q_jobs, kv_jobs;
  std::vector<int32_t> q_off, q_list, kv_off, kv_list;
  std::vector<TileRef> tiles;
};

// Key positions in the lists: contiguous K/V -- key rows of the K / V tensors; paged --
// sequence-local key indices (the kernels map them through row `seq` of the page table),
// with each item's page count in `pad` and each dQ job's valid keys in `rows`.
void build_bwd(const Shape& s, const std::vector<std::vector<int32_t>>& cnts, int num_sms, BwdLists& bl) {
  const int g = s.hq / s.hkv;
  std::vector<int64_t> q_cost, kv_cost, q_group, kv_group;
  for (int b = 0; b < s.B; ++b) {
    const int lq = s.lq[b], lk = s.lk[b];
    const int n_qt = (lq + kTile - 1) / kTile, n_kt = (lk + kTile - 1) / kTile;
    const int32_t kbase = s.paged ? 0 : s.koff[b], npg = s.paged ? (lk + s.ps - 1) / s.ps : 0;
    const std::vector<int32_t>& cnt = cnts[b];
    // How every (query tile, key tile) is masked, the same for all heads; partial tiles are
    // numbered in row-major order. Row lists serve the dQ items, column lists the dK/dV items.
    std::vector<int32_t> row_off(size_t(n_qt) + 1, 0), col_off(size_t(n_kt) + 1, 0);
    std::vector<int32_t> tab(size_t(n_qt) * n_kt, kMaskNone);
    for (int qt = 0; qt < n_qt; ++qt)
      for (int kt = 0; kt < n_kt; ++kt) {
        const int64_t rows = std::min(kTile, lq - qt * kTile), cols = std::min(kTile, lk - kt * kTile);
        const int32_t k = classify(cnt[size_t(qt) * n_kt + kt], rows * cols);
        int32_t m = kMaskNone;
        if (k == kClassFull && (kt + 1) * kTile <= lk && (qt + 1) * kTile <= lq) {
          m = kMaskFull;
        } else if (k != kClassEmpty) {
          m = int32_t(bl.tiles.size());
          bl.tiles.push_back(TileRef{b, qt, kt, m});
        }
        tab[size_t(qt) * n_kt + kt] = m;
        if (m != kMaskNone) {
          row_off[qt + 1]++;
          col_off[kt + 1]++;
        }
      }
    for (int qt = 0; qt < n_qt; ++qt) row_off[qt + 1] += row_off[qt];
    for (int kt = 0; kt < n_kt; ++kt) col_off[kt + 1] += col_off[kt];
    std::vector<int32_t> row_kt(row_off[n_qt]), col_qt(col_off[n_kt]);
    {
      std::vector<int32_t> rf(row_off.begin(), row_off.end() - 1), cf(col_off.begin(), col_off.end() - 1);
      for (int qt = 0; qt < n_qt; ++qt)
        for (int kt = 0; kt < n_kt; ++kt)
          if (tab[size_t(qt) * n_kt + kt] != kMaskNone) {
            row_kt[rf[qt]++] = kt;
            col_qt[cf[kt]++] = qt;
          }
    }
    const size_t nnz = row_kt.size();
    bl.q_jobs.reserve(bl.q_jobs.size() + nnz + n_qt);
    bl.kv_jobs.reserve(bl.kv_jobs.size() + size_t(s.hq) * nnz + size_t(s.hkv) * n_kt);
    // A dQ job names a key tile and its mask only (the dQ kernel takes the head from the
    // item), so the query heads of one query tile share one list.
    std::vector<int32_t> q_start(size_t(n_qt), -1), q_count(size_t(n_qt), 0);
    for (int kh = 0; kh < s.hkv; ++kh) {
      // dQ items
      for (int h = kh * g; h < (kh + 1) * g; ++h)
        for (int qt = 0; qt < n_qt; ++qt) {
          BwdItem it{b, kh, h, s.qoff[b] + qt * kTile, std::min(kTile, lq - qt * kTile), int32_t(bl.q_jobs.size()), 0,
                     npg};
          if (q_start[qt] >= 0) {
            it.job_start = q_start[qt];
            it.job_count = q_count[qt];
          } else {
            for (int32_t e = row_off[qt]; e < row_off[qt + 1]; ++e) {
              const int kt = row_kt[e];
              bl.q_jobs.push_back(BwdJob{kbase + kt * kTile, tab[size_t(qt) * n_kt + kt], h, std::min(kTile, lk - kt * kTile)});
            }
            if (bl.q_jobs.size() == size_t(it.job_start))   // no key anywhere: one hidden job writes dq = 0
              bl.q_jobs.push_back(BwdJob{kbase, kMaskNone, h, 0});
            it.job_count = int32_t(bl.q_jobs.size()) - it.job_start;
            q_start[qt] = it.job_start;
            q_count[qt] = it.job_count;
          }
          q_cost.push_back(it.job_count + 2);
          q_group.push_back(int64_t(b) * s.hkv + kh);
          bl.q_items.push_back(it);
        }
      // dK/dV items
      for (int kt = 0; kt < n_kt; ++kt) {
        BwdItem it{b, kh, kh * g, kbase + kt * kTile, std::min(kTile, lk - kt * kTile),
                   int32_t(bl.kv_jobs.size()), 0, npg};
        for (int h = kh * g; h < (kh + 1) * g; ++h)
          for (int32_t e = col_off[kt]; e < col_off[kt + 1]; ++e) {
            const int qt = col_qt[e];
            bl.kv_jobs.push_back(BwdJob{s.qoff[b] + qt * kTile, tab[size_t(qt) * n_kt + kt], h,
                                        std::min(kTile, lq - qt * kTile)});
          }
        if (bl.kv_jobs.size() == size_t(it.job_start))   // no query sees the tile: dk = dv = 0
          bl.kv_jobs.push_back(BwdJob{s.qoff[b], kMaskNone, kh * g, 0});
        it.job_count = int32_t(bl.kv_jobs.size()) - it.job_start;
        kv_cost.push_back(it.job_count + 2);
        kv_group.push_back(int64_t(b) * s.hkv + kh);
        bl.kv_items.push_back(it);
      }
    }
  }
  assign_lpt(q_cost, q_group, num_sms, bl.q_off, bl.q_list);
  assign_lpt(kv_cost, kv_group, num_sms, bl.kv_off, bl.kv_list);
}

// 32 x 32 bit matrix (word i = row i, bit k = column k) transposed in place: the off-diagonal
// halves, quarters, ... of the rows are swapped in five rounds of masked shifts.
void transpose32(uint32_t a[32]) {
  uint32_t m = 0x0000FFFFu;
  for (int j = 16; j != 0; j >>= 1, m ^= (m << j)) {
    for (int k = 0; k < 32; k = (k + j + 1) & ~j) {
      const uint32_t t = ((a[k] >> j) ^ a[k + j]) & m;
      a[k] ^= t << j;
      a[k + j] ^= t;
    }
  }
}

// Row-major 2 KiB tile (row r: 4 words, bit c = key c) -> the transposed tile (row c, bit r),
// as 4 x 4 blocks of 32 x 32 bits.
void transpose_tile(const uint32_t* src, uint32_t* dst) {
  for (int rb = 0; rb < 4; ++rb)
    for (int cb = 0; cb < 4; ++cb) {
      uint32_t a[32];
      for (int i = 0; i < 32; ++i) a[i] = src[4 * (32 * rb + i) + cb];
      transpose32(a);
      for (int j = 0; j < 32; ++j) dst[4 * (32 * cb + j) + rb] = a[j];
    }
}

attn_status_t plan_backward(const attn_mask_desc_t* mask, const Shape& s, RowSource& src, int num_sms,
                            cudaStream_t stream, attn_plan_t* plan) {
  if (s.paged) {
    // The gradient of a cache page shared by two sequences would be the sum of both
    // sequences' contributions; the dK/dV kernel writes each page's rows from one work item,
    // so every page a sequence reads (entries in [0, num_pages)) must belong to it alone.
    std::vector<int32_t> pt(size_t(s.B) * s.maxp);
    if (!pt.empty()) {
      cudaError_t e = cudaMemcpyAsync(pt.data(), plan->page_table, pt.size() * 4, cudaMemcpyDeviceToHost, stream);
      if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
      if (e != cudaSuccess) return ATTN_ERR_CUDA;
    }
    std::vector<uint8_t> seen(size_t(s.npages), 0);
    for (int b = 0; b < s.B; ++b)
      for (int i = 0; i < (s.lk[b] + s.ps - 1) / s.ps; ++i) {
        const int32_t pg = pt[size_t(b) * s.maxp + i];
        if (pg < 0 || pg >= s.npages) continue;
        if (seen[size_t(pg)]) return ATTN_ERR_UNSUPPORTED;
        seen[size_t(pg)] = 1;
      }
  }
  std::vector<std::vector<int32_t>> cnts(s.B);
  if (mask->kind == ATTN_MASK_CUSTOM) {
    attn_status_t st = custom_counts(mask, s, kTile, stream, cnts);
    if (st != ATTN_OK) return st;
  } else {
    for (int b = 0; b < s.B; ++b) {
      src.prepare(b);
      count_sequence(src, b, s, kTile, cnts[b]);
    }
  }
  BwdLists bl;
  build_bwd(s, cnts, num_sms, bl);
  const size_t nt = bl.tiles.size();
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  const size_t o_qi = take(bl.q_items.size() * sizeof(BwdItem)), o_qj = take(bl.q_jobs.size() * sizeof(BwdJob)),
               o_qo = take(bl.q_off.size() * 4), o_ql = take(bl.q_list.size() * 4),
               o_ki = take(bl.kv_items.size() * sizeof(BwdItem)), o_kj = take(bl.kv_jobs.size() * sizeof(BwdJob)),
               o_ko = take(bl.kv_off.size() * 4), o_kl = take(bl.kv_list.size() * 4),
               o_mq = take(nt * kMaskTileBytes), o_mk = take(nt * kMaskTileBytes),
               o_dl = take(size_t(std::max<int64_t>(1, s.total_q)) * s.hq * sizeof(float));
  void* ws = nullptr;
  cudaError_t e = cudaMalloc(&ws, off);
  if (e != cudaSuccess) return cuda_status(e);
  char* base = static_cast<char*>(ws);
  std::vector<uint32_t> qmaj(nt * (kMaskTileBytes / 4)), kmaj(nt * (kMaskTileBytes / 4));
  // the lists go up straight from their vectors (the block-dense lists are ~46 MB: a host
  // staging copy would double the host traffic); the padding between them is zeroed on the
  // device
  e = cudaMemsetAsync(base, 0, o_mq, stream);
  const struct {
    size_t dst;
    const void* src;
    size_t bytes;
  } parts[] = {{o_qi, bl.q_items.data(), bl.q_items.size() * sizeof(BwdItem)},
               {o_qj, bl.q_jobs.data(), bl.q_jobs.size() * sizeof(BwdJob)},
               {o_qo, bl.q_off.data(), bl.q_off.size() * 4},
               {o_ql, bl.q_list.data(), bl.q_list.size() * 4},
               {o_ki, bl.kv_items.data(), bl.kv_items.size() * sizeof(BwdItem)},
               {o_kj, bl.kv_jobs.data(), bl.kv_jobs.size() * sizeof(BwdJob)},
               {o_ko, bl.kv_off.data(), bl.kv_off.size() * 4},
               {o_kl, bl.kv_list.data(), bl.kv_list.size() * 4}};
  for (const auto& pt : parts)
    if (e == cudaSuccess && pt.bytes)
      e = cudaMemcpyAsync(base + pt.dst, pt.src, pt.bytes, cudaMemcpyHostToDevice, stream);
  attn_status_t st = cuda_status(e);
  if (st == ATTN_OK && nt) {
    if (mask->kind == ATTN_MASK_CUSTOM) {
      st = custom_repack(mask, s, kTile, bl.tiles, reinterpret_cast<uint4*>(base + o_mq), stream);
      if (st == ATTN_OK)
        st = cuda_status(cudaMemcpy(qmaj.data(), base + o_mq, nt * kMaskTileBytes, cudaMemcpyDeviceToHost));
    } else {
      int cur = -1;
      for (const TileRef& t : bl.tiles) {
        if (t.seq != cur) {
          src.prepare(t.seq);
          cur = t.seq;
        }
        write_mask_tile(src, s, kTile, t, qmaj.data() + size_t(t.idx) * (kMaskTileBytes / 4));
      }
      st = cuda_status(cudaMemcpyAsync(base + o_mq, qmaj.data(), nt * kMaskTileBytes, cudaMemcpyHostToDevice, stream));
    }
    for (size_t i = 0; st == ATTN_OK && i < nt; ++i)
      transpose_tile(qmaj.data() + i * (kMaskTileBytes / 4), kmaj.data() + i * (kMaskTileBytes / 4));
    if (st == ATTN_OK)
      st = cuda_status(cudaMemcpyAsync(base + o_mk, kmaj.data(), nt * kMaskTileBytes, cudaMemcpyHostToDevice, stream));
  }
  if (st == ATTN_OK) st = cuda_status(cudaStreamSynchronize(stream));
  if (st != ATTN_OK) {
    cudaFree(ws);
    return st;
  }
  plan->has_bwd = true;
  plan->bws = ws;
  plan->bq_ctas = int32_t(bl.q_off.size()) - 1;
  plan->bkv_ctas = int32_t(bl.kv_off.size()) - 1;
  plan->d_bq_items = reinterpret_cast<const BwdItem*>(base + o_qi);
  plan->d_bq_jobs = reinterpret_cast<const BwdJob*>(base + o_qj);
  plan->d_bq_cta_off = reinterpret_cast<const int32_t*>(base + o_qo);
  plan->d_bq_cta_items = reinterpret_cast<const int32_t*>(base + o_ql);
  plan->d_bkv_items = reinterpret_cast<const BwdItem*>(base + o_ki);
  plan->d_bkv_jobs = reinterpret_cast<const BwdJob*>(base + o_kj);
  plan->d_bkv_cta_off = reinterpret_cast<const int32_t*>(base + o_ko);
  plan->d_bkv_cta_items = reinterpret_cast<const int32_t*>(base + o_kl);
  plan->d_bmask_q = reinterpret_cast<const uint4*>(base + o_mq);
  plan->d_bmask_k = reinterpret_cast<const uint4*>(base + o_mk);
  plan->d_bdelta = reinterpret_cast<float*>(base + o_dl);
  return ATTN_OK;
}

// Problem shape and kernel shape of a plan from the validated problem.
void fill_meta(const Shape& s, const attn_problem_t* problem, attn_plan_t& m) {
  m.batch = s.B;
  m.hq = s.hq;
  m.hkv = s.hkv;
  m.d = s.d;
  m.scale = s.scale;
  m.paged = s.paged;
  m.page_size = s.ps;
  m.max_pages = s.maxp;
  m.num_pages = s.npages;
  m.page_table = s.paged ? problem->page_table : nullptr;
  m.total_q = s.total_q;
  m.total_kv_rows = s.total_kv_rows;
  choose_shape(s, m);
}

attn_status_t plan_impl(const attn_problem_t* problem, const attn_mask_desc_t* mask, cudaStream_t stream,
                        attn_plan_t** out_plan, bool with_bwd = false) {
  if (!out_plan) return ATTN_ERR_INVALID_ARG;
  *out_plan = nullptr;
  Shape s;
  attn_status_t st = validate_problem(problem, s);
  if (st != ATTN_OK) return st;
  st = validate_mask(mask, s);
  if (st != ATTN_OK) return st;

  int dev = 0, num_sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return ATTN_ERR_CUDA;

  auto plan = new attn_plan_t();
  // frees the plan and what it holds on every early return and on an exception
  struct Guard {
    attn_plan_t* p;
    ~Guard() {
      if (!p) return;
      if (p->ws) cudaFree(p->ws);
      if (p->bws) cudaFree(p->bws);
      delete p;
    }
  } guard{plan};
  plan->device = dev;
  fill_meta(s, problem, *plan);
  const int R = plan->R;

  std::vector<std::vector<int32_t>> cnts(s.B);
  RowSource src(mask, s);
  if (mask->kind == ATTN_MASK_CUSTOM) {
    st = custom_counts(mask, s, R, stream, cnts);
    if (st != ATTN_OK) return st;
  } else {
    for (int b = 0; b < s.B; ++b) {
      src.prepare(b);
      count_sequence(src, b, s, R, cnts[b]);
    }
  }
  for (int b = 0; b < s.B; ++b) report_classes(cnts[b], s.lq[b], s.lk[b], R, plan->classes, plan->stats);

  WorkList wl;
  build_work(s, R, plan->hp, plan->nq, cnts, num_sms / plan->cluster, wl);
  plan->ctas = int32_t(wl.cta_off.size()) - 1;   // work units: CTAs, or CTA pairs
  plan->vt_keys = s.paged ? 0 : vt_offsets(s)[s.B];
  work_stats(*plan, wl, plan->stats);

  const Staging lay = layout(wl, s.d, s.B);
  plan->stats.workspace_bytes = int64_t(lay.total);
  std::vector<char> host(lay.off_tiles, 0);
  std::memcpy(host.data() + lay.off_items, wl.items.data(), wl.items.size() * sizeof(WorkItem));
  std::memcpy(host.data() + lay.off_jobs, wl.jobs.data(), wl.jobs.size() * sizeof(Job));
  std::memcpy(host.data() + lay.off_cta_off, wl.cta_off.data(), wl.cta_off.size() * sizeof(int32_t));
  std::memcpy(host.data() + lay.off_cta_items, wl.cta_items.data(), wl.cta_items.size() * sizeof(int32_t));
  {
    const std::vector<int32_t> vt_off = vt_offsets(s);
    std::vector<int32_t> cu_k(size_t(s.B) + 1, 0);
    for (int b = 0; b < s.B; ++b) cu_k[b + 1] = s.paged ? 0 : s.koff[b] + s.lk[b];
    if (!s.paged && s.B > 0) cu_k[0] = s.koff[0];
    std::memcpy(host.data() + lay.off_seq, cu_k.data(), cu_k.size() * sizeof(int32_t));
    std::memcpy(host.data() + lay.off_seq + cu_k.size() * sizeof(int32_t), vt_off.data(), vt_off.size() * sizeof(int32_t));
  }
  std::vector<uint32_t> tiles;
  if (mask->kind != ATTN_MASK_CUSTOM && !wl.mask_tiles.empty()) {
    tiles.resize(wl.mask_tiles.size() * (kMaskTileBytes / 4));
    int cur = -1;
    for (const TileRef& t : wl.mask_tiles) {
      if (t.seq != cur) {
        src.prepare(t.seq);
        cur = t.seq;
      }
      write_mask_tile(src, s, R, t, tiles.data() + size_t(t.idx) * (kMaskTileBytes / 4));
    }
  }

  e = cudaMalloc(&plan->ws, lay.total);
  if (e != cudaSuccess) {
    plan->ws = nullptr;
    return cuda_status(e);
  }
  plan->ws_bytes = lay.total;
  char* base = static_cast<char*>(plan->ws);
  plan->d_status = reinterpret_cast<int32_t*>(base);
  plan->d_items = reinterpret_cast<const WorkItem*>(base + lay.off_items);
  plan->d_jobs = reinterpret_cast<const Job*>(base + lay.off_jobs);
  plan->d_cta_off = reinterpret_cast<const int32_t*>(base + lay.off_cta_off);
  plan->d_cta_items = reinterpret_cast<const int32_t*>(base + lay.off_cta_items);
  plan->d_mask_tiles = reinterpret_cast<const uint4*>(base + lay.off_tiles);
  plan->d_cu_k = reinterpret_cast<const int32_t*>(base + lay.off_seq);
  plan->d_vt_off = plan->d_cu_k + (s.B + 1);
  if (!wl.merge.empty()) {
    plan->d_merge = reinterpret_cast<const MergeTile*>(base + lay.off_merge);
    plan->n_merge = int32_t(wl.merge.size());
    plan->d_part_lse = reinterpret_cast<float*>(base + lay.off_part_lse);
    plan->d_part_o = reinterpret_cast<float*>(base + lay.off_part_o);
  }
  e = cudaMemcpyAsync(base, host.data(), host.size(), cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess && !tiles.empty())
    e = cudaMemcpyAsync(base + lay.off_tiles, tiles.data(), tiles.size() * 4, cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess && !wl.merge.empty())
    e = cudaMemcpyAsync(base + lay.off_merge, wl.merge.data(), wl.merge.size() * sizeof(MergeTile),
                        cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  st = cuda_status(e);
  if (st == ATTN_OK && mask->kind == ATTN_MASK_CUSTOM)
    st = custom_repack(mask, s, R, wl.mask_tiles, reinterpret_cast<uint4*>(base + lay.off_tiles), stream);
  if (st == ATTN_OK && with_bwd) st = plan_backward(mask, s, src, num_sms, stream, plan);
  if (st != ATTN_OK) return st;
  guard.p = nullptr;
  *out_plan = plan;
  return ATTN_OK;
}

}  // namespace

// Host-only planning for attn_masked_fwd_noalloc (analytic kinds): the same validation,
// classification, work list and mask tiles as attn_plan, written into host bytes in the
// workspace layout instead of a device allocation.
attn_status_t mfa_plan_host(const attn_problem_t* problem, const attn_mask_desc_t* mask, int num_sms,
                            mfa_host_plan* out) {
  try {
    if (mask && mask->kind == ATTN_MASK_CUSTOM) return ATTN_ERR_UNSUPPORTED;
    Shape s;
    attn_status_t st = validate_problem(problem, s);
    if (st != ATTN_OK) return st;
    st = validate_mask(mask, s);
    if (st != ATTN_OK) return st;
    attn_plan_t& m = out->meta;
    fill_meta(s, problem, m);
    const int R = m.R;
    std::vector<std::vector<int32_t>> cnts(s.B);
    RowSource src(mask, s);
    for (int b = 0; b < s.B; ++b) {
      src.prepare(b);
      count_sequence(src, b, s, R, cnts[b]);
    }
    WorkList wl;
    build_work(s, R, m.hp, m.nq, cnts, num_sms / m.cluster, wl, /*allow_split=*/false);
    m.ctas = int32_t(wl.cta_off.size()) - 1;
    const Staging lay = layout(wl, s.d, s.B);
    out->off_items = lay.off_items;
    out->off_jobs = lay.off_jobs;
    out->off_cta_off = lay.off_cta_off;
    out->off_cta_items = lay.off_cta_items;
    out->off_tiles = lay.off_tiles;
    out->bytes.assign(lay.total, 0);
    char* h = out->bytes.data();
    std::memcpy(h + lay.off_items, wl.items.data(), wl.items.size() * sizeof(WorkItem));
    std::memcpy(h + lay.off_jobs, wl.jobs.data(), wl.jobs.size() * sizeof(Job));
    std::memcpy(h + lay.off_cta_off, wl.cta_off.data(), wl.cta_off.size() * sizeof(int32_t));
    std::memcpy(h + lay.off_cta_items, wl.cta_items.data(), wl.cta_items.size() * sizeof(int32_t));
    int cur = -1;
    for (const TileRef& t : wl.mask_tiles) {
      if (t.seq != cur) {
        src.prepare(t.seq);
        cur = t.seq;
      }
      write_mask_tile(src, s, R, t,
                      reinterpret_cast<uint32_t*>(h + lay.off_tiles + size_t(t.idx) * kMaskTileBytes));
    }
    return ATTN_OK;
  } catch (const std::bad_alloc&) {
    return ATTN_ERR_OOM;
  } catch (...) {
    return ATTN_ERR_INVALID_ARG;
  }
}

extern "C" {

attn_status_t attn_test_transpose_mask_tile(const uint32_t* src, uint32_t* dst) {
  if (!src || !dst) return ATTN_ERR_INVALID_ARG;
  transpose_tile(src, dst);
  return ATTN_OK;
}

attn_status_t attn_plan_bwd_dry_run(const attn_problem_t* problem, const attn_mask_desc_t* mask, int32_t num_sms,
                                    attn_bwd_stats_t* stats) {
  try {
    if (!stats || num_sms <= 0) return ATTN_ERR_INVALID_ARG;
    if (mask && mask->kind == ATTN_MASK_CUSTOM) return ATTN_ERR_UNSUPPORTED;
    Shape s;
    attn_status_t st = validate_problem(problem, s, /*need_device_ptrs=*/false);
    if (st != ATTN_OK) return st;
    st = validate_mask(mask, s);
    if (st != ATTN_OK) return st;
    std::vector<std::vector<int32_t>> cnts(s.B);
    RowSource src(mask, s);
    for (int b = 0; b < s.B; ++b) {
      src.prepare(b);
      count_sequence(src, b, s, kTile, cnts[b]);
    }
    BwdLists bl;
    build_bwd(s, cnts, num_sms, bl);
    attn_bwd_stats_t out{};
    auto side = [](const std::vector<BwdItem>& items, const std::vector<int32_t>& off,
                   const std::vector<int32_t>& list, int64_t& n_items, int64_t& n_jobs, int32_t& ctas,
                   int64_t& cost, int64_t& max_cta, int64_t& max_item) {
      n_items = int64_t(items.size());
      for (const BwdItem& it : items) {
        n_jobs += it.job_count;
        cost += it.job_count + 2;
        max_item = std::max<int64_t>(max_item, it.job_count + 2);
      }
      ctas = int32_t(off.size()) - 1;
      for (int32_t c = 0; c < ctas; ++c) {
        int64_t load = 0;
        for (int32_t e = off[c]; e < off[c + 1]; ++e) load += items[size_t(list[e])].job_count + 2;
        max_cta = std::max(max_cta, load);
      }
    };
    side(bl.q_items, bl.q_off, bl.q_list, out.dq_items, out.dq_jobs, out.dq_ctas, out.dq_cost, out.dq_max_cta_cost,
         out.dq_max_item_cost);
    side(bl.kv_items, bl.kv_off, bl.kv_list, out.dkv_items, out.dkv_jobs, out.dkv_ctas, out.dkv_cost,
         out.dkv_max_cta_cost, out.dkv_max_item_cost);
    out.mask_tiles = int64_t(bl.tiles.size());
    *stats = out;
    return ATTN_OK;
  } catch (const std::bad_alloc&) {
    return ATTN_ERR_OOM;
  } catch (...) {
    return ATTN_ERR_INVALID_ARG;
  }
}

attn_status_t attn_plan_dry_run(const attn_problem_t* problem, const attn_mask_desc_t* mask, int32_t num_sms,
                                attn_plan_stats_t* stats) {
  try {
    if (!stats || num_sms <= 0) return ATTN_ERR_INVALID_ARG;
    if (mask && mask->kind == ATTN_MASK_CUSTOM) return ATTN_ERR_UNSUPPORTED;
    Shape s;
    attn_status_t st = validate_problem(problem, s, /*need_device_ptrs=*/false);
    if (st != ATTN_OK) return st;
    st = validate_mask(mask, s);
    if (st != ATTN_OK) return st;
    attn_plan_t m;
    fill_meta(s, problem, m);
    attn_plan_stats_t out{};
    std::vector<std::vector<int32_t>> cnts(s.B);
    RowSource src(mask, s);
    for (int b = 0; b < s.B; ++b) {
      src.prepare(b);
      count_sequence(src, b, s, m.R, cnts[b]);
      report_classes(cnts[b], s.lq[b], s.lk[b], m.R, m.classes, out);
    }
    WorkList wl;
    build_work(s, m.R, m.hp, m.nq, cnts, num_sms / m.cluster, wl);
    m.ctas = int32_t(wl.cta_off.size()) - 1;
    m.vt_keys = s.paged ? 0 : vt_offsets(s)[s.B];
    work_stats(m, wl, out);
    out.workspace_bytes = int64_t(layout(wl, s.d, s.B).total);
    *stats = out;
    return ATTN_OK;
  } catch (const std::bad_alloc&) {
    return ATTN_ERR_OOM;
  } catch (...) {
    return ATTN_ERR_INVALID_ARG;
  }
}

attn_status_t attn_plan(const attn_problem_t* problem, const attn_mask_desc_t* mask, attn_stream_t stream,
                        attn_plan_t** out_plan) {
  try {
    return plan_impl(problem, mask, reinterpret_cast<cudaStream_t>(stream), out_plan);
  } catch (const std::bad_alloc&) {
    return ATTN_ERR_OOM;
  } catch (...) {
    return ATTN_ERR_INVALID_ARG;
  }
}

attn_status_t attn_plan_bwd(const attn_problem_t* problem, const attn_mask_desc_t* mask, attn_stream_t stream,
                            attn_plan_t** out_plan) {
  try {
    return plan_impl(problem, mask, reinterpret_cast<cudaStream_t>(stream), out_plan, /*with_bwd=*/true);
  } catch (const std::bad_alloc&) {
    return ATTN_ERR_OOM;
  } catch (...) {
    return ATTN_ERR_INVALID_ARG;
  }
}

// The plan's workspace lives on the device it was made on: its kernels run there only.
static bool on_plan_device(const attn_plan_t* plan) {
  int dev = -1;
  return cudaGetDevice(&dev) == cudaSuccess && dev == plan->device;
}

attn_status_t attn_masked_bwd(const attn_plan_t* plan, const void* q, const void* k, const void* v, const void* out,
                              const float* lse, const void* dout, const float* dlse, void* dq, void* dk, void* dv,
                              attn_stream_t stream) {
  if (!plan || !plan->has_bwd || !on_plan_device(plan)) return ATTN_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, out, lse, dout, dq, dk, dv};
  for (const void* p : ptrs)
    if (!p || (reinterpret_cast<uintptr_t>(p) & 15u)) return ATTN_ERR_INVALID_ARG;
  if (dlse && (reinterpret_cast<uintptr_t>(dlse) & 3u)) return ATTN_ERR_INVALID_ARG;
  return mfa_launch_backward(plan, q, k, v, out, lse, dout, dlse, dq, dk, dv, reinterpret_cast<cudaStream_t>(stream));
}

attn_status_t attn_fp8_transpose_v(const attn_plan_t* plan, const void* v, void* vt, int64_t ldv,
                                   attn_stream_t stream) {
  if (!plan || plan->paged || !v || !vt || ldv < plan->vt_keys || ldv % 16 != 0 || !on_plan_device(plan))
    return ATTN_ERR_INVALID_ARG;
  if (plan->d % 32 != 0) return ATTN_ERR_UNSUPPORTED;
  return mfa_transpose_v(plan, v, vt, ldv, reinterpret_cast<cudaStream_t>(stream));
}

attn_status_t attn_masked_fwd_fp8(const attn_plan_t* plan, const void* q, const void* k, const void* vt, int64_t ldv,
                                  float q_scale, float k_scale, float v_scale, void* out, float* lse,
                                  attn_stream_t stream) {
  if (!plan || !on_plan_device(plan)) return ATTN_ERR_INVALID_ARG;
  if ((plan->d != 128 && plan->d != 256) || plan->paged) return ATTN_ERR_UNSUPPORTED;
  const void* ptrs[] = {q, k, vt, out};
  for (const void* p : ptrs)
    if (!p || (reinterpret_cast<uintptr_t>(p) & 15u)) return ATTN_ERR_INVALID_ARG;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return ATTN_ERR_INVALID_ARG;
  if (ldv < plan->vt_keys || ldv % 16 != 0) return ATTN_ERR_INVALID_ARG;
  for (float x : {q_scale, k_scale, v_scale})
    if (!(x > 0.f) || std::isinf(x)) return ATTN_ERR_INVALID_ARG;
  return mfa_launch_forward_fp8(plan, q, k, vt, ldv, q_scale, k_scale, v_scale, out, lse,
                                reinterpret_cast<cudaStream_t>(stream));
}

attn_status_t attn_masked_fwd(const attn_plan_t* plan, const void* q, const void* k, const void* v, void* out,
                              float* lse, attn_stream_t stream) {
  if (!plan || !on_plan_device(plan)) return ATTN_ERR_INVALID_ARG;
  if (plan->total_q == 0) return ATTN_OK;
  if (!q || !k || !v || !out) return ATTN_ERR_INVALID_ARG;
  auto mis = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) != 0; };
  if (mis(q) || mis(k) || mis(v) || mis(out) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3)))
    return ATTN_ERR_INVALID_ARG;
  return mfa_launch_forward(plan, q, k, v, out, lse, reinterpret_cast<cudaStream_t>(stream));
}

attn_status_t attn_plan_get_tile_classes(const attn_plan_t* plan, uint8_t* host_dst, size_t n, size_t* n_needed) {
  if (!plan) return ATTN_ERR_INVALID_ARG;
  if (n_needed) *n_needed = plan->classes.size();
  if (n && !host_dst) return ATTN_ERR_INVALID_ARG;
  std::memcpy(host_dst, plan->classes.data(), std::min(n, plan->classes.size()));
  return ATTN_OK;
}

attn_status_t attn_plan_get_stats(const attn_plan_t* plan, attn_plan_stats_t* stats) {
  if (!plan || !stats) return ATTN_ERR_INVALID_ARG;
  *stats = plan->stats;
  return ATTN_OK;
}

attn_status_t attn_plan_check_status(const attn_plan_t* plan, attn_stream_t stream) {
  if (!plan) return ATTN_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int32_t host[4] = {0, 0, 0, 0};
  cudaError_t e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemcpy(host, plan->d_status, sizeof(host), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(plan->d_status, 0, sizeof(host));
  if (e != cudaSuccess) return ATTN_ERR_CUDA;
  if (host[0] != 0) return ATTN_ERR_TIMEOUT;
  return ATTN_OK;
}

attn_status_t attn_plan_set_debug(attn_plan_t* plan, int32_t flags, int64_t timeout_ns) {
  if (!plan || flags < 0 || timeout_ns < 0) return ATTN_ERR_INVALID_ARG;
  plan->debug_flags = flags;
  plan->timeout_ns = timeout_ns > 0 ? timeout_ns : 2000000000LL;
  return ATTN_OK;
}

attn_status_t attn_plan_destroy(attn_plan_t* plan) {
  if (!plan) return ATTN_OK;
  cudaError_t e = cudaSuccess;
  if (plan->ws) e = cudaFree(plan->ws);
  if (plan->bws) {
    const cudaError_t e2 = cudaFree(plan->bws);
    if (e == cudaSuccess) e = e2;
  }
  delete plan;
  return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

attn_status_t attn_classify_host(const attn_problem_t* problem, const attn_mask_desc_t* mask, uint8_t* classes,
                                 size_t n, size_t* n_needed, int64_t* unmasked_pairs) {
  try {
    Shape s;
    attn_status_t st = validate_problem(problem, s, /*need_device_ptrs=*/false);
    if (st != ATTN_OK) return st;
    st = validate_mask(mask, s);
    if (st != ATTN_OK) return st;
    if (mask->kind == ATTN_MASK_CUSTOM) return ATTN_ERR_UNSUPPORTED;
    RowSource src(mask, s);
    std::vector<uint8_t> out;
    attn_plan_stats_t stats{};
    std::vector<int32_t> cnt;
    for (int b = 0; b < s.B; ++b) {
      src.prepare(b);
      count_sequence(src, b, s, kTile, cnt);
      report_classes(cnt, s.lq[b], s.lk[b], kTile, out, stats);
    }
    if (n_needed) *n_needed = out.size();
    if (unmasked_pairs) *unmasked_pairs = stats.unmasked_pairs;
    if (classes) std::memcpy(classes, out.data(), std::min(n, out.size()));
    return ATTN_OK;
  } catch (const std::bad_alloc&) {
    return ATTN_ERR_OOM;
  } catch (...) {
    return ATTN_ERR_INVALID_ARG;
  }
}

const char* attn_status_string(attn_status_t status) {
  switch (status) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID_ARG: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported configuration";
    case ATTN_ERR_MASK_TOO_SMALL: return "custom mask buffer too small for the lengths";
    case ATTN_ERR_OOM: return "out of device memory";
    case ATTN_ERR_CUDA: return "CUDA runtime error";
    case ATTN_ERR_TIMEOUT: return "a bounded wait in the kernel expired";
    case ATTN_ERR_TOO_LARGE: return "the plan exceeds the fixed scratch of attn_masked_fwd_noalloc";
    default: return "unknown status";
  }
}

}  // extern "C"
