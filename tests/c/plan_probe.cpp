// The host planner (attn_plan.cpp) built against host-memory stand-ins for the CUDA runtime
// calls it makes, so that a test can run attn_plan() without a GPU and read the workspace it
// would upload: the work items, their jobs and the 2 KiB partial-tile masks. The kernel
// launchers are stubs that report "unsupported"; CUSTOM masks (scanned by a device kernel)
// therefore fail to plan here. Test infrastructure only.
#include <cstdlib>
#include <cstring>

#include <cuda_runtime.h>

extern "C" {
cudaError_t cudaMalloc(void** p, size_t n) {
  *p = std::malloc(n ? n : 1);
  if (!*p) return cudaErrorMemoryAllocation;
  std::memset(*p, 0xCD, n);   // "uninitialised device memory": nothing may rely on its value
  return cudaSuccess;
}
cudaError_t cudaFree(void* p) {
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
  *d = 0;
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
namespace mfa {
cudaError_t launch_custom_count(const uint32_t*, const CustomSeq*, const CountTask*, int, int, int32_t*,
                                cudaStream_t) {
  return cudaErrorNotSupported;
}
cudaError_t launch_custom_repack(const uint32_t*, const CustomSeq*, const RepackTask*, int, int, uint4*,
                                 cudaStream_t) {
  return cudaErrorNotSupported;
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
