// Internal types shared by the host planner (attn_plan.cpp), the forward kernel
// (attn_fwd.cu) and the CUSTOM-mask scan (attn_custom.cu). Not part of the ABI.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>
#include <vector>

#include "attn.h"

namespace mfa {

constexpr int kTile = 128;          // query rows and keys per tile, and per classification tile
constexpr int kMaskTileBytes = 2048;  // 128 rows x 128 bits

// mask field of a Job
constexpr int32_t kMaskFull = -1;   // tile fully visible: no mask arithmetic
constexpr int32_t kMaskNone = -2;   // tile fully hidden for this query tile (pairing filler)

// One unit of forward work: up to two 128-row query tiles that share one key/value
// head and iterate over the same key tiles. Row r of tile t is query head
// head[t] + r / R at token tok[t] + r % R, valid when r % R < rows[t]
// (R = 128 / heads_per_tile).
struct alignas(16) WorkItem {
  int32_t seq;
  int32_t kv_head;
  int32_t k_base;      // contiguous: first key row of the sequence; paged: seq * max_pages_per_seq
  int32_t kv_len;      // valid keys of the sequence
  int32_t tok[2];
  int32_t rows[2];
  int32_t head[2];
  int32_t job_start;
  int32_t job_count;
  int32_t npages;      // paged: pages that hold the sequence's keys
  int32_t part;        // -1: write out / lse; else query tile t writes partial slot part + t
  int32_t vt_base;     // contiguous: first column of the sequence in a transposed V (128-aligned)
  int32_t pad;
};
static_assert(sizeof(WorkItem) == 64, "WorkItem layout");

// A query tile whose key tiles were split over several work items (split-KV): its rows'
// partial results sit in slots slot0, slot0 + stride, ... (nsplit of them) and are merged
// into out / lse by the merge kernel. Rows as in WorkItem (tile row r: token tok + r % R,
// head head + r / R, valid when r % R < rows).
struct alignas(16) MergeTile {
  int32_t tok, head, rows;
  int32_t slot0, nsplit, stride;
  int32_t pad[2];
};
static_assert(sizeof(MergeTile) == 32, "MergeTile layout");

// Partial-result slots: 128 rows x head_dim fp32 (out / l) and 128 fp32 lse values each.
constexpr int kSlotRows = 128;
// Most key ranges one query tile is split into (the merge kernel keeps that many weights per row).
constexpr int kMaxSplits = 256;

// One key tile of a work item and, per query tile, how to mask it.
struct alignas(16) Job {
  int32_t k_tile;
  int32_t mask[2];     // kMaskFull, kMaskNone or the index of a 2 KiB mask tile
  int32_t pad;
};
static_assert(sizeof(Job) == 16, "Job layout");

// ---- backward work lists (attn_plan_bwd) -------------------------------------------------
// dQ items: one 128-row query tile of one query head against its non-empty key tiles.
// dK/dV items: one 128-key tile of one key/value head against every (query head of its
// group, query tile) that sees it. Tiles here are always 128 rows of one head.
struct alignas(16) BwdItem {
  int32_t seq, kv_head;
  int32_t head;        // dQ: the query head
  int32_t tok;         // dQ: first query token of the tile; dK/dV: first key row of the tile
                       // (paged: sequence-local key index)
  int32_t rows;        // valid rows of the tile (queries, or keys)
  int32_t job_start, job_count;
  int32_t npages;      // paged K/V: pages of the sequence's keys (0 for contiguous K/V)
};
static_assert(sizeof(BwdItem) == 32, "BwdItem layout");

struct alignas(16) BwdJob {
  int32_t tok;         // dQ: first key row of the key tile (paged: sequence-local key index);
                       // dK/dV: first query token of the query tile
  int32_t mask;        // kMaskFull, kMaskNone, or a mask tile (dQ: query-major; dK/dV: key-major)
  int32_t head;        // dK/dV: the query head
  int32_t rows;        // dK/dV: valid query rows of the query tile; dQ: valid keys of the key tile
};
static_assert(sizeof(BwdJob) == 16, "BwdJob layout");

// ---- CUSTOM mask scan on the device ----------------------------------------------------
struct CustomSeq {
  int64_t word_off;    // first word of the sequence's packed mask
  int64_t cnt_off;     // first count of the sequence in the count array
  int32_t lq, lk;
  int32_t n_rb, n_kt;  // row blocks of R rows, key tiles of 128
};
struct CountTask { int32_t seq, rb, kt0, pad; };   // one row block x up to 32 key tiles
struct RepackTask { int32_t seq, rb, kt, idx; };    // one mask tile to write

cudaError_t launch_custom_count(const uint32_t* bits, const CustomSeq* seqs, const CountTask* tasks,
                                int ntasks, int R, int32_t* counts, cudaStream_t stream);
cudaError_t launch_custom_repack(const uint32_t* bits, const CustomSeq* seqs, const RepackTask* tasks,
                                 int ntasks, int R, uint4* tiles, cudaStream_t stream);

}  // namespace mfa

struct attn_plan {
  // problem
  int32_t batch = 0, hq = 0, hkv = 0, d = 0;
  float scale = 0.f;
  bool paged = false;
  int32_t page_size = 0, max_pages = 0, num_pages = 0;
  const int32_t* page_table = nullptr;   // device
  int64_t total_q = 0, total_kv_rows = 0;
  // kernel shape
  int32_t nq = 1;        // query tiles per work item
  int32_t cluster = 1;   // CTAs per work item (2: the cluster-pair kernel, one tile per CTA)
  int32_t hp = 1;        // heads packed per query tile
  int32_t R = 128;       // rows per head in a query tile
  int32_t ctas = 0;
  // host results
  std::vector<uint8_t> classes;
  attn_plan_stats_t stats{};
  // device workspace (one allocation)
  void* ws = nullptr;
  size_t ws_bytes = 0;
  int32_t* d_status = nullptr;
  const mfa::WorkItem* d_items = nullptr;
  const mfa::Job* d_jobs = nullptr;
  const int32_t* d_cta_off = nullptr;
  const int32_t* d_cta_items = nullptr;
  const uint4* d_mask_tiles = nullptr;
  // contiguous K/V: per sequence [B + 1] key offsets and 128-aligned transposed-V column offsets
  const int32_t* d_cu_k = nullptr;
  const int32_t* d_vt_off = nullptr;
  int64_t vt_keys = 0;
  // split-KV: partial slots and the tiles to merge (none when nothing was split)
  float* d_part_o = nullptr;
  float* d_part_lse = nullptr;
  const mfa::MergeTile* d_merge = nullptr;
  int32_t n_merge = 0;
  // backward (attn_plan_bwd; one more workspace allocation)
  bool has_bwd = false;
  void* bws = nullptr;
  int32_t bq_ctas = 0, bkv_ctas = 0;
  const mfa::BwdItem* d_bq_items = nullptr;
  const mfa::BwdJob* d_bq_jobs = nullptr;
  const int32_t* d_bq_cta_off = nullptr;
  const int32_t* d_bq_cta_items = nullptr;
  const mfa::BwdItem* d_bkv_items = nullptr;
  const mfa::BwdJob* d_bkv_jobs = nullptr;
  const int32_t* d_bkv_cta_off = nullptr;
  const int32_t* d_bkv_cta_items = nullptr;
  const uint4* d_bmask_q = nullptr;   // query-major 2 KiB tiles (row = query, bits = keys)
  const uint4* d_bmask_k = nullptr;   // the same tiles transposed (row = key, bits = queries)
  float* d_bdelta = nullptr;          // [total_q][hq]: dout . out per row
  // debug hooks
  int32_t debug_flags = 0;
  int64_t timeout_ns = 2000000000LL;
  int device = 0;
};

// Host-only plan used by attn_masked_fwd_noalloc: the bytes attn_plan would upload, laid
// out as [status | items | jobs | cta_off | cta_items | mask tiles] from offset 0 (attn_plan.cpp).
struct mfa_host_plan {
  attn_plan_t meta;            // problem and kernel shape; device pointers left unset
  std::vector<char> bytes;
  size_t off_items = 0, off_jobs = 0, off_cta_off = 0, off_cta_items = 0, off_tiles = 0;
};
attn_status_t mfa_plan_host(const attn_problem_t* problem, const attn_mask_desc_t* mask, int num_sms,
                            mfa_host_plan* out);

// forward launcher (attn_fwd.cu)
attn_status_t mfa_launch_forward(const attn_plan_t* plan, const void* q, const void* k, const void* v,
                                 void* out, float* lse, cudaStream_t stream);

// e4m3 forward and the V transpose it reads (attn_fwd.cu)
attn_status_t mfa_launch_forward_fp8(const attn_plan_t* plan, const void* q, const void* k, const void* vt,
                                     int64_t ldv, float q_scale, float k_scale, float v_scale, void* out, float* lse,
                                     cudaStream_t stream);
attn_status_t mfa_transpose_v(const attn_plan_t* plan, const void* v, void* vt, int64_t ldv, cudaStream_t stream);

// backward launcher (attn_bwd.cu)
attn_status_t mfa_launch_backward(const attn_plan_t* plan, const void* q, const void* k, const void* v,
                                  const void* out, const float* lse, const void* dout, const float* dlse,
                                  void* dq, void* dk, void* dv, cudaStream_t stream);
