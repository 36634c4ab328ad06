// The host planner (attn_plan.cpp) built against host-memory stand-ins for the CUDA runtime
// calls it makes, so that a test can run attn_plan() without a GPU and read the workspace it
// would upload: the work items, their jobs and the 2 KiB partial-tile masks. The attention
// launchers are stubs that report "unsupported"; the CUSTOM mask scan runs as host code
// written from the scan kernels' contracts. Test infrastructure only.
#include <cstdlib>
#include <cstring>

#include <cuda_runtime.h>

static int g_mallocs_left = -1;   // >= 0: that many more allocations succeed, then they fail
static int g_live = 0;            // device allocations not freed yet
static int g_device = 0;          // the "current device"

extern "C" {
void probe_fail_malloc_after(int n) { g_mallocs_left = n; }
void probe_set_device(int d) { g_device = d; }
int probe_live_allocations() { return g_live; }
cudaError_t cudaMalloc(void** p, size_t n) {
  if (g_mallocs_left == 0) {
    *p = nullptr;
    return cudaErrorMemoryAllocation;
  }
  if (g_mallocs_left > 0) --g_mallocs_left;
  *p = std::malloc(n ? n : 1);
  if (!*p) return cudaErrorMemoryAllocation;
  ++g_live;
  std::memset(*p, 0xCD, n);   // "uninitialised device memory": nothing may rely on its value
  return cudaSuccess;
}
cudaError_t cudaFree(void* p) {
  if (p) --g_live;
  std::free(p);
  return cudaSuccess;
}
cudaError_t cudaMemcpyAsync(void* d, const void* s, size_t n, cudaMemcpyKind, cudaStream_t) {
  std::memcpy(d, s, n);
  return cudaSuccess;
}
cudaError_t cudaMemcpy(void* d, const void* s, size_t n, cudaMemcpyKind) {
  std::memcpy(d, s, n);
  return cudaSuccess;
}
cudaError_t cudaMemsetAsync(void* d, int v, size_t n, cudaStream_t) {
  std::memset(d, v, n);
  return cudaSuccess;
}
cudaError_t cudaMemset(void* d, int v, size_t n) {
  std::memset(d, v, n);
  return cudaSuccess;
}
cudaError_t cudaStreamSynchronize(cudaStream_t) { return cudaSuccess; }
cudaError_t cudaGetDevice(int* d) {
  *d = g_device;
  return cudaSuccess;
}
cudaError_t cudaDeviceGetAttribute(int* v, cudaDeviceAttr, int) {
  *v = 148;
  return cudaSuccess;
}
}

#include "attn_plan.cpp"

attn_status_t mfa_launch_forward(const attn_plan_t*, const void*, const void*, const void*, void*, float*,
                                 cudaStream_t) {
  return ATTN_ERR_UNSUPPORTED;
}
attn_status_t mfa_launch_forward_fp8(const attn_plan_t*, const void*, const void*, const void*, int64_t, float, float,
                                     float, void*, float*, cudaStream_t) {
  return ATTN_ERR_UNSUPPORTED;
}
attn_status_t mfa_transpose_v(const attn_plan_t*, const void*, void*, int64_t, cudaStream_t) {
  return ATTN_ERR_UNSUPPORTED;
}
attn_status_t mfa_launch_backward(const attn_plan_t*, const void*, const void*, const void*, const void*, const float*,
                                  const void*, const float*, void*, void*, void*, cudaStream_t) {
  return ATTN_ERR_UNSUPPORTED;
}
// Host versions of the two CUSTOM-mask kernels, from their stated contracts (the device
// kernels themselves are checked on the GPU): count = visible keys of every (R-row block,
// 128-key tile) of a task's 32 key tiles; repack = 128 rows x 4 words per tile, query row
// rb * R + r % R, bits past L_k or past the sequence's rows cleared.
namespace mfa {
namespace {
uint32_t row_word(const uint32_t* bits, const CustomSeq& s, int64_t i, int64_t w) {
  const int64_t W = (int64_t(s.lk) + 31) / 32;
  if (i >= s.lq || w >= W) return 0u;
  const int64_t rem = int64_t(s.lk) - 32 * w;
  const uint32_t valid = rem >= 32 ? 0xffffffffu : ((1u << rem) - 1u);
  return bits[s.word_off + i * W + w] & valid;
}
}  // namespace
cudaError_t launch_custom_count(const uint32_t* bits, const CustomSeq* seqs, const CountTask* tasks, int ntasks,
                                int R, int32_t* counts, cudaStream_t) {
  for (int n = 0; n < ntasks; ++n) {
    const CountTask& t = tasks[n];
    const CustomSeq& s = seqs[t.seq];
    for (int kt = t.kt0; kt < std::min(s.n_kt, t.kt0 + 32); ++kt) {
      int32_t c = 0;
      for (int64_t i = int64_t(t.rb) * R; i < std::min<int64_t>(s.lq, int64_t(t.rb + 1) * R); ++i)
        for (int j = 0; j < 4; ++j) c += __builtin_popcount(row_word(bits, s, i, int64_t(kt) * 4 + j));
      counts[s.cnt_off + int64_t(t.rb) * s.n_kt + kt] = c;
    }
  }
  return cudaSuccess;
}
cudaError_t launch_custom_repack(const uint32_t* bits, const CustomSeq* seqs, const RepackTask* tasks, int ntasks,
                                 int R, uint4* tiles, cudaStream_t) {
  for (int n = 0; n < ntasks; ++n) {
    const RepackTask& t = tasks[n];
    const CustomSeq& s = seqs[t.seq];
    for (int r = 0; r < 128; ++r) {
      const int64_t i = int64_t(t.rb) * R + r % R;
      uint32_t w[4];
      for (int j = 0; j < 4; ++j) w[j] = row_word(bits, s, i, int64_t(t.kt) * 4 + j);
      tiles[int64_t(t.idx) * 128 + r] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
  return cudaSuccess;
}
}  // namespace mfa

extern "C" {
// The forward workspace of a plan: items [n_items] (64-byte WorkItem), jobs (16-byte Job,
// indexed by the items), mask tiles [n_tiles][128 rows][4 words]; rows per head R, heads per
// tile and query tiles per item.
int probe_forward(const attn_plan_t* p, const void** items, const void** jobs, const void** tiles,
                  int64_t* n_items, int64_t* n_tiles, int32_t* R, int32_t* hp, int32_t* nq) {
  if (!p) return 1;
  *items = p->d_items;
  *jobs = p->d_jobs;
  *tiles = p->d_mask_tiles;
  *n_items = p->stats.work_items;
  *n_tiles = p->stats.mask_tiles;
  *R = p->R;
  *hp = p->hp;
  *nq = p->nq;
  return 0;
}

// Split-KV: the merge list (32-byte MergeTile: tok, head, rows, slot0, nsplit, stride).
int probe_merge(const attn_plan_t* p, const void** merge, int64_t* n) {
  if (!p) return 1;
  *merge = p->d_merge;
  *n = p->n_merge;
  return 0;
}

// The host plan of the allocation-free entry (the bytes it copies into its fixed array):
// the same pointers as probe_forward, into a plan object the caller frees with
// probe_host_plan_free.
void* probe_host_plan(const attn_problem_t* problem, const attn_mask_desc_t* mask, int* status, const void** items,
                      const void** jobs, const void** tiles, int64_t* n_items, int64_t* n_tiles, int64_t* bytes) {
  auto* hp = new mfa_host_plan();
  *status = int(mfa_plan_host(problem, mask, 148, hp));
  if (*status != ATTN_OK) {
    delete hp;
    return nullptr;
  }
  const char* b = hp->bytes.data();
  *items = b + hp->off_items;
  *jobs = b + hp->off_jobs;
  *tiles = b + hp->off_tiles;
  *n_items = reinterpret_cast<const int32_t*>(b + hp->off_cta_off)[hp->meta.ctas];   // every item listed once
  *n_tiles = (hp->bytes.size() - hp->off_tiles) / kMaskTileBytes;
  *bytes = int64_t(hp->bytes.size());
  return hp;
}
void probe_host_plan_free(void* hp) { delete static_cast<mfa_host_plan*>(hp); }

// The backward lists of an attn_plan_bwd() plan: dQ and dK/dV items (32-byte BwdItem), their
// jobs (16-byte BwdJob) and the query-major / key-major mask tiles.
int probe_backward(const attn_plan_t* p, const void** q_items, const void** q_jobs, const void** kv_items,
                   const void** kv_jobs, const void** mask_q, const void** mask_k, int64_t* n_q, int64_t* n_kv) {
  if (!p || !p->has_bwd) return 1;
  *q_items = p->d_bq_items;
  *q_jobs = p->d_bq_jobs;
  *kv_items = p->d_bkv_items;
  *kv_jobs = p->d_bkv_jobs;
  *mask_q = p->d_bmask_q;
  *mask_k = p->d_bmask_k;
  *n_q = p->d_bq_cta_off ? reinterpret_cast<const int32_t*>(p->d_bq_cta_off)[p->bq_ctas] : 0;
  *n_kv = p->d_bkv_cta_off ? reinterpret_cast<const int32_t*>(p->d_bkv_cta_off)[p->bkv_ctas] : 0;
  return 0;
}
}
