// Device scan of a bit-packed CUSTOM mask ("Custom mask slows down attention.",
// flashinfer #724: the custom mask is handed over as a bit-packed array).
//
// count: visible keys of every (R-row block, 128-key tile) of every sequence, read with
//        fully coalesced 128-byte row segments (a warp reads 32 consecutive words of a
//        row, i.e. 8 key tiles, per instruction). The host turns the counts into
//        empty / full / partial classes.
// repack: every tile the forward has to mask is rewritten in the tile-transposed layout:
//        128 rows x 16 bytes, row r's 128 bits at byte 16 r, so that the forward reads
//        one row's mask with a single 16-byte load per thread (a warp reads 512
//        contiguous bytes). Bits outside the sequence are cleared; for R < 128 the R
//        query rows are repeated 128 / R times (one copy per packed head).
#include "attn_internal.h"

namespace mfa {
namespace {

__device__ __forceinline__ uint32_t valid_bits(int64_t word, int32_t lk) {
  const int64_t rem = int64_t(lk) - word * 32;
  if (rem <= 0) return 0u;
  return rem >= 32 ? 0xffffffffu : ((1u << rem) - 1u);
}

__global__ void __launch_bounds__(128) custom_count_kernel(const uint32_t* __restrict__ bits,
                                                           const CustomSeq* __restrict__ seqs,
                                                           const CountTask* __restrict__ tasks, int R,
                                                           int32_t* __restrict__ counts) {
  const CountTask t = tasks[blockIdx.x];
  const CustomSeq s = seqs[t.seq];
  const int64_t W = (int64_t(s.lk) + 31) / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t w_begin = int64_t(t.kt0) * 4;
  const int64_t w_end = min(W, w_begin + 128);
  int64_t widx[4];
  uint32_t vm[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    widx[j] = w_begin + lane + 32 * j;
    vm[j] = widx[j] < w_end ? valid_bits(widx[j], s.lk) : 0u;
  }
  uint32_t acc[4] = {0u, 0u, 0u, 0u};
  const int r0 = t.rb * R, r1 = min(s.lq, r0 + R);
  for (int i = r0 + warp; i < r1; i += 4) {
    const uint32_t* row = bits + s.word_off + int64_t(i) * W;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (vm[j]) acc[j] += __popc(__ldg(row + widx[j]) & vm[j]);
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], 1);
    acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], 2);
  }
  __shared__ uint32_t part[4][32];
  if ((lane & 3) == 0) {
#pragma unroll
    for (int j = 0; j < 4; ++j) part[warp][lane / 4 + 8 * j] = acc[j];
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    const int kt = t.kt0 + int(threadIdx.x);
    if (kt < s.n_kt) {
      const uint32_t c = part[0][threadIdx.x] + part[1][threadIdx.x] + part[2][threadIdx.x] + part[3][threadIdx.x];
      counts[s.cnt_off + int64_t(t.rb) * s.n_kt + kt] = int32_t(c);
    }
  }
}

__global__ void __launch_bounds__(128) custom_repack_kernel(const uint32_t* __restrict__ bits,
                                                            const CustomSeq* __restrict__ seqs,
                                                            const RepackTask* __restrict__ tasks, int R,
                                                            uint4* __restrict__ tiles) {
  const RepackTask t = tasks[blockIdx.x];
  const CustomSeq s = seqs[t.seq];
  const int64_t W = (int64_t(s.lk) + 31) / 32;
  const int r = threadIdx.x;
  const int i = t.rb * R + (r % R);
  uint32_t w[4] = {0u, 0u, 0u, 0u};
  if (i < s.lq) {
    const uint32_t* row = bits + s.word_off + int64_t(i) * W;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t wi = int64_t(t.kt) * 4 + j;
      if (wi < W) w[j] = __ldg(row + wi) & valid_bits(wi, s.lk);
    }
  }
  tiles[int64_t(t.idx) * 128 + r] = make_uint4(w[0], w[1], w[2], w[3]);
}

}  // namespace

cudaError_t launch_custom_count(const uint32_t* bits, const CustomSeq* seqs, const CountTask* tasks, int ntasks,
                                int R, int32_t* counts, cudaStream_t stream) {
  if (ntasks <= 0) return cudaSuccess;
  custom_count_kernel<<<ntasks, 128, 0, stream>>>(bits, seqs, tasks, R, counts);
  return cudaGetLastError();
}

cudaError_t launch_custom_repack(const uint32_t* bits, const CustomSeq* seqs, const RepackTask* tasks, int ntasks,
                                 int R, uint4* tiles, cudaStream_t stream) {
  if (ntasks <= 0) return cudaSuccess;
  custom_repack_kernel<<<ntasks, 128, 0, stream>>>(bits, seqs, tasks, R, tiles);
  return cudaGetLastError();
}

}  // namespace mfa
