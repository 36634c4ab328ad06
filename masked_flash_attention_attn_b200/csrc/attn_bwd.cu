// Masked attention backward for sm_100a (B200): dQ, dK and dV of the forward in attn_fwd.cu.
//
// With p_ij = exp(scale q_i . k_j - lse_i) on visible pairs (0 elsewhere), dp_ij = dout_i . v_j,
// delta_i = dout_i . out_i and ds_ij = p_ij (dp_ij - delta_i):
//     dq_i = scale sum_j ds_ij k_j,   dk_j = scale sum_i ds_ij q_i,   dv_j = sum_i p_ij dout_i,
// dk and dv of a key/value head summed over the query heads that read it. Three kernels:
//   bwd_delta_kernel    delta_i for every (row, query head): d / 8 lanes per row.
//   dQ kernel           one persistent CTA per SM over dQ items (a 128-row query tile of one
//                       query head and its non-empty key tiles): S = Q K^T and dP = dO V^T
//                       into TMEM, the elementwise warpgroups turn them into dS (bf16, written
//                       over S), then dQ += dS K accumulates in TMEM.
//   dK/dV kernel        one persistent CTA per SM over dK/dV items (a 128-key tile of one
//                       key/value head and every (query head, query tile) that sees it):
//                       S^T = K Q^T and dP^T = V dO^T into TMEM, the warpgroups write P^T
//                       and dS^T (bf16) over them, then dV += P^T dO and dK += dS^T Q accumulate in
//                       TMEM.
// Both recompute P from the forward's lse instead of storing it. Warp roles: warp 0 TMA
// producer; warp 1 issues the S (S^T) MMAs, warp 3 the dP (dP^T) MMAs and warp 2 the
// accumulating MMAs (dQ, or dV and dK), one thread each, so that no MMA waits behind another
// kind's dependency in a shared issue order; warps 4-11 two elementwise warpgroups, one TMEM
// lane (= one tile row) per thread, the first warpgroup on columns 0..63 of every job and the
// second on columns 64..127. Tiles are 128 rows of one head, 64-column boxes with the
// 128-byte swizzle; rings of tile slots stream the per-job operands (dQ: a ring of K tiles,
// held until the dQ MMA, and a shallower one of V tiles; dK/dV: one ring of Q and dO tiles).
// A job is one 128 x 128 block, its S and dP MMAs M = 128, N = 128: the tensor core reads
// 8 KiB of shared memory per 128 x 128 x 16 step, the rate its 64-cycle step can take
// (narrower N re-reads A for every N block). The hand-offs are per operand, so each MMA
// starts as soon as the TMEM it reads or overwrites allows:
//   dQ:    S slots 0 / 1 (TMEM columns 0 and 128), one dP slot (256), dQ (384). S of job g+1
//          runs while the warpgroups work on job g; dP of job g+1 once they have read dP of
//          job g (they read it first); dQ += dS K once they have written dS over S.
//   dK/dV: two job slots (TMEM columns 0 and 128), dV (256) and dK (256 + D). Job g uses
//          slot g % 2 three times over: S^T, which the warpgroups read into registers; then
//          dP^T, computed over it; then P^T and dS^T (bf16), which the warpgroups write over
//          dP^T and dV += P^T dO, dK += dS^T Q read. Two jobs are in flight: S^T of job g+1
//          runs while the warpgroups work on job g.
// dQ: bf16 dS pairs of columns 0..63 go to TMEM columns 0..31 of the S slot and those of
// columns 64..127 to 64..95; dK/dV: P^T pairs to columns 0..31 / 64..95 of the slot and dS^T
// pairs to 32..63 / 96..127. Each warpgroup writes only columns it has already read. Every
// mbarrier wait is bounded as in the forward. At head_dim 256 (Bwd256Cfg) the tiles are too
// large for this layout: the streamed operands come as half-tiles, one thread issues a job's
// MMAs in order, and dK / dV take two passes, one per head-dim half of the accumulators.

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "attn_internal.h"

namespace mfa {
namespace {

#include "device_common.cuh"

// The elementwise loops work on packed fp32 pairs (one f32x2 instruction per two elements):
// the two warps of each sub-partition are limited by issue slots and the MUFU exponentials.
__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// 2^x of a packed pair (MUFU).
__device__ __forceinline__ uint64_t exp2_pair(uint64_t x) {
  float x0, x1;
  unpk2(x, x0, x1);
  return pk2(ex2(x0), ex2(x1));
}

// Two bf16 of a packed pair (lower element in the low half).
__device__ __forceinline__ uint32_t pack_bf16x2(uint64_t v) {
  float a, b;
  unpk2(v, a, b);
  return pack_bf16(a, b);
}

struct BwdParams {
  CUtensorMap tm_a;   // per item:  dQ: Q    dK/dV: K
  CUtensorMap tm_b;   // per item:  dQ: dO   dK/dV: V
  CUtensorMap tm_c;   // per job:   dQ: K    dK/dV: Q
  CUtensorMap tm_d;   // per job:   dQ: V    dK/dV: dO
  const BwdItem* items;
  const BwdJob* jobs;
  const int32_t* cta_off;
  const int32_t* cta_items;
  const uint4* mask_tiles;
  const float* lse;     // [total_q][hq], natural log
  const float* delta;   // [total_q][hq]
  __nv_bfloat16* g0;    // dQ: dq;  dK/dV: dk
  __nv_bfloat16* g1;    // dK/dV: dv
  int32_t* status;
  int32_t hq, hkv;
  int32_t debug_flags;   // bit 0: skip the first item's per-item loads (testing the timeout path)
  int32_t dhalf;         // head_dim 256 dK/dV pass: the half of the head dimension accumulated
  const int32_t* page_table;   // paged K/V: [batch][maxp] pages of each sequence's keys
  int32_t page_size, num_pages, maxp;
  float scale, scale_log2;
  int64_t timeout_ns;
};

// Shared-memory layout, TMEM columns and mbarriers of the two kernels. A job is one
// 128 x 128 tile pair, S and dP (dQ) or S^T and dP^T (dK/dV) computed as M = 128, N = 128
// MMAs; the accumulators take D (dQ) or 2 D (dV, dK) TMEM columns.
template <int D_, bool DKV_, bool PAGED_ = false>
struct BwdCfg {
  static constexpr int D = D_;
  static constexpr bool DKV = DKV_;
  static constexpr bool PAGED = PAGED_;   // K / V from a paged cache
  static constexpr int NBOX = D / 64;                  // 64-column boxes per tile
  static constexpr int BOX_BYTES = 128 * 128;          // 128 rows x 128 bytes
  static constexpr int TILE_BYTES = NBOX * BOX_BYTES;  // one 128-row tile of one head
  // Ring tile slots. dK/dV: one ring of Q and dO tiles, two per job. dQ: a ring of K tiles
  // and a ring of V tiles -- K is held until the job's dQ MMA, V only until its dP MMA, so the
  // K ring is the deeper one.
  static constexpr int STAGES = D == 128 ? 4 : 8;
  static constexpr int KST = D == 128 ? 3 : 5, VST = D == 128 ? 2 : 3;
  static constexpr int RING = DKV ? STAGES : KST + VST;
  // TMEM: dQ -- S slots at 0 and 128, dP at 256, dQ at 384; dK/dV -- two job slots at 0 and
  // 128 (S^T, then dP^T over it, then P^T and dS^T), dV at 256, dK at 256 + D
  static constexpr int NS = 2;                         // S (dQ) or job (dK/dV) slots
  static constexpr int TM_S = 0, TM_P = 256, TM_ACC = DKV ? 256 : 384;
  static constexpr int OFF_A = 0, OFF_B = TILE_BYTES, OFF_RING = 2 * TILE_BYTES;
  static constexpr int OFF_ROWV = OFF_RING + RING * TILE_BYTES;  // dK/dV: per warp 128 lse2 + 128 delta
  static constexpr int OFF_BAR = OFF_ROWV + (DKV ? 8 * 2 * 128 * 4 : 0);
  // dQ:    SFULL[s] S of slot s computed, DPFULL[0] dP computed, READ[0] dP read by the
  //        warpgroups, DSREADY[s] dS written, SFREE[s] the dQ MMA of slot s completed.
  // dK/dV: SFULL[s] S^T of slot s computed, READ[s] S^T read by the warpgroups, DPFULL[s]
  //        dP^T computed (over S^T), DSREADY[s] P^T and dS^T written (over dP^T), SFREE[s]
  //        the dV and dK MMAs of slot s completed.
  static constexpr int B_AFULL = 0, B_AEMPTY = 1, B_RFULL = 2, B_REMPTY = B_RFULL + RING,
                       B_SFULL = B_REMPTY + RING, B_DPFULL = B_SFULL + NS, B_READ = B_DPFULL + NS,
                       B_DSREADY = B_READ + NS, B_SFREE = B_DSREADY + NS, B_ACCFULL = B_SFREE + NS,
                       B_ACCEMPTY = B_ACCFULL + 1, B_DRAIN = B_ACCEMPTY + 1, B_DRAIN2 = B_DRAIN + 1,
                       B_DRAIN3 = B_DRAIN2 + 1, NBAR = B_DRAIN3 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;       // [0] TMEM base, [1] abort flag
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;   // + slack to align the base to 1 KiB
  static constexpr int THREADS = 384;
  static constexpr int EW = 256;                            // elementwise threads (two warpgroups)
  static constexpr uint32_t IDESC_SS =  // M=128, N=128, bf16 x bf16 -> fp32, both K-major
      (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(128 >> 3) << 17) | (uint32_t(128 >> 4) << 24);
  static constexpr uint32_t IDESC_TS =  // M=128, N=D, A from TMEM, B MN-major
      (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | (uint32_t(D >> 3) << 17) | (uint32_t(128 >> 4) << 24);
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(TM_ACC + (DKV ? 2 * D : D) <= 512, "TMEM budget");
};

enum : int32_t {
  kBwdWaitAEmpty = 0x200, kBwdWaitREmpty, kBwdWaitAFull, kBwdWaitRFull, kBwdWaitPFull, kBwdWaitAccEmpty,
  kBwdWaitSFull, kBwdWaitAccFull, kBwdWaitSFree, kBwdWaitDpFull, kBwdWaitDpRead, kBwdWaitDsReady, kBwdWaitDpFree
};

// C[128 x 128] (TMEM, fp32) = A[128 x D] . B[128 x D]^T, both whole tiles, K-major in
// shared memory.
template <int D>
__device__ __forceinline__ void mma_tile_ss(uint32_t d, uint32_t a_smem, uint32_t b_smem, uint32_t idesc) {
  if constexpr (D == 128) mma_ss_x8_k128(d, desc_of(desc_lo(a_smem, 16)), desc_of(desc_lo(b_smem, 16)), idesc, 0u);
  else mma_ss_x4_k64(d, desc_of(desc_lo(a_smem, 16)), desc_of(desc_lo(b_smem, 16)), idesc, 0u);
}

// C[128 x D] (+)= A[128 x 128] . B[128 x D]: A is bf16 in TMEM, its 128 K columns (64 TMEM
// columns) in two runs of 32 -- columns a .. a + 31 (K 0..63, written by the first
// elementwise warpgroup) and a + 64 .. a + 95 (K 64..127, the second) -- and B a whole tile
// in shared memory, MN-major.
__device__ __forceinline__ void mma_tile_ts(uint32_t d, uint32_t a, uint32_t b_smem, uint32_t idesc, uint32_t acc) {
  const uint64_t b = desc_of(desc_lo(b_smem, 128 * 128));
  asm volatile(
      "{\n\t.reg .pred p, t;\n\t.reg .b32 ta, bl, bh;\n\t.reg .b64 bx;\n\t"
      "setp.ne.b32 p, %4, 0;\n\tsetp.eq.u32 t, 0, 0;\n\t"
      "mov.b64 {bl, bh}, %2;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t"
      "add.u32 ta, %1, 8;\n\tadd.u32 bl, bl, 128;\n\tmov.b64 bx, {bl, bh};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], bx, %3, t;\n\t"
      "add.u32 ta, %1, 16;\n\tadd.u32 bl, bl, 128;\n\tmov.b64 bx, {bl, bh};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], bx, %3, t;\n\t"
      "add.u32 ta, %1, 24;\n\tadd.u32 bl, bl, 128;\n\tmov.b64 bx, {bl, bh};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], bx, %3, t;\n\t"
      "add.u32 ta, %1, 64;\n\tadd.u32 bl, bl, 128;\n\tmov.b64 bx, {bl, bh};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], bx, %3, t;\n\t"
      "add.u32 ta, %1, 72;\n\tadd.u32 bl, bl, 128;\n\tmov.b64 bx, {bl, bh};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], bx, %3, t;\n\t"
      "add.u32 ta, %1, 80;\n\tadd.u32 bl, bl, 128;\n\tmov.b64 bx, {bl, bh};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], bx, %3, t;\n\t"
      "add.u32 ta, %1, 88;\n\tadd.u32 bl, bl, 128;\n\tmov.b64 bx, {bl, bh};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], bx, %3, t;\n\t"
      "}" ::"r"(d),
      "r"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

// NC columns of a 128-row tile of gradients from TMEM (fp32, times `mul`) to global memory as
// bf16 (dst: this row's first column of the run).
template <int NC>
__device__ __forceinline__ void store_grad_cols(uint32_t t_acc, float mul, bool valid, __nv_bfloat16* dst) {
#pragma unroll 1
  for (int cc = 0; cc < NC / 32; ++cc) {
    uint32_t o[32];
    tmem_ld32x32(t_acc + cc * 32, o);
    tmem_wait_ld();
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e)
      pk[e] = pack_bf16(__uint_as_float(o[2 * e]) * mul, __uint_as_float(o[2 * e + 1]) * mul);
    if (valid) {
      uint4* q = reinterpret_cast<uint4*>(dst + cc * 32);
      q[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      q[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
      q[2] = make_uint4(pk[8], pk[9], pk[10], pk[11]);
      q[3] = make_uint4(pk[12], pk[13], pk[14], pk[15]);
    }
  }
}

// delta[r][h] = dout[r][h] . out[r][h] - dlse[r][h] (fp32; dlse may be null) over the rows
// r = (token, head) of D bf16 values. With a gradient on lse, ds = p (dp - delta) picks up
// + p dlse. A row is read by D / 8 lanes, 16 bytes of each tensor per lane (both 16-byte
// aligned), and every lane keeps four rows' loads in flight: one warp per row with 4-byte
// loads left the read at under half of the HBM rate.
__device__ __forceinline__ float dot8_bf16(const uint4& a, const uint4& b) {
  const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&aw[i]));
    const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bw[i]));
    acc = fmaf(x.x, y.x, acc);
    acc = fmaf(x.y, y.y, acc);
  }
  return acc;
}

template <int D>
__global__ void bwd_delta_kernel(const __nv_bfloat16* __restrict__ out, const __nv_bfloat16* __restrict__ dout,
                                 const float* __restrict__ dlse, float* __restrict__ delta, int64_t rows) {
  constexpr int L = D / 8, RPW = 32 / L, U = 4;   // lanes per row, rows per warp pass, passes in flight
  const int lane = threadIdx.x & 31, sub = lane % L, grp = lane / L;
  const int64_t warp0 = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (int64_t(gridDim.x) * blockDim.x) >> 5;
  for (int64_t base = warp0 * (RPW * U); base < rows; base += nwarps * (RPW * U)) {   // warp-uniform
    uint4 o[U], g[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t r = base + u * RPW + grp;
      o[u] = g[u] = make_uint4(0u, 0u, 0u, 0u);
      if (r < rows) {
        o[u] = __ldg(reinterpret_cast<const uint4*>(out + r * D) + sub);
        g[u] = __ldg(reinterpret_cast<const uint4*>(dout + r * D) + sub);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float acc = dot8_bf16(o[u], g[u]);
#pragma unroll
      for (int m = L / 2; m > 0; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
      const int64_t r = base + u * RPW + grp;
      if (sub == 0 && r < rows) delta[r] = dlse ? acc - dlse[r] : acc;
    }
  }
}

// Row r's 128 mask bits of a job: the packed partial tile, all ones (fully visible) or all
// zeros (a filler job that sees nothing).
__device__ __forceinline__ uint4 row_bits(const uint4* __restrict__ tiles, int mi, int r) {
  if (mi >= 0) return __ldg(tiles + int64_t(mi) * 128 + r);
  return mi == kMaskNone ? make_uint4(0u, 0u, 0u, 0u) : make_uint4(0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu);
}

// Paged K/V: one key tile (128 keys from tile-local row 0) of sequence `seq` into `dst`, the
// tile's pages issued by lanes 0 .. 128 / page_size - 1 of the calling warp (one TMA issue
// stream per page). Pages past the sequence's last, or outside the cache, read as zeros.
template <int NBOX>
__device__ __forceinline__ void load_paged_tile(const BwdParams& p, const CUtensorMap* tm, uint32_t dst, int seq,
                                                int key0, int npages, int kv_head, uint32_t bar, int lane) {
  const int ps = p.page_size, ppt = 128 / ps;
  if (lane < ppt) {
    const int idx = key0 / ps + lane;
    const int32_t page = idx < npages ? __ldg(p.page_table + int64_t(seq) * p.maxp + idx) : -1;
    int32_t row = p.num_pages * ps;   // fully out of bounds: the box reads zeros
    if (page >= 0 && page < p.num_pages) row = page * ps;
    for (int c = 0; c < NBOX; ++c) tma_load_3d(dst + c * 128 * 128 + lane * ps * 128, tm, c * 64, kv_head, row, bar);
  }
}

// Rows r0 .. 127 of a tile of NBOX 64-column boxes set to zero by one thread (a paged cache
// holds stale rows past a sequence's last key in its last page; a zero row times a zero
// score weight must stay zero in the MMAs), then made visible to the tensor core.
template <int NBOX>
__device__ __forceinline__ void zero_tile_rows(uint32_t tile, int r0) {
  for (int i = 0; i < (128 - r0) * NBOX * 8; ++i) {
    const int row = r0 + i / (NBOX * 8), rem = i % (NBOX * 8);
    asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(tile + uint32_t((rem >> 3) * 16384 + row * 128 +
                                                                                   (rem & 7) * 16)),
                 "r"(0u)
                 : "memory");
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ================================ dQ ================================
template <class C>
__global__ void __launch_bounds__(C::THREADS, 1) masked_attn_bwd_dq_kernel(const __grid_constant__ BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem_raw + (sbase - raw) + C::OFF_MISC);
  const uint32_t bar0 = sbase + C::OFF_BAR;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Guard guard{smem_u32(misc + 1), 0u, p.status, p.timeout_ns};
#define BAR(i) (bar0 + 8u * uint32_t(i))
  if (tid == 0) {
    mbar_init(BAR(C::B_AFULL), 1);
    mbar_init(BAR(C::B_AEMPTY), 2);   // both S-side issuers commit
    for (int s = 0; s < C::RING; ++s) {
      mbar_init(BAR(C::B_RFULL + s), 1);
      mbar_init(BAR(C::B_REMPTY + s), 1);
    }
    for (int b = 0; b < C::NS; ++b) {
      mbar_init(BAR(C::B_SFULL + b), 1);
      mbar_init(BAR(C::B_DSREADY + b), C::EW);
      mbar_init(BAR(C::B_SFREE + b), 1);
    }
    mbar_init(BAR(C::B_DPFULL), 1);
    mbar_init(BAR(C::B_READ), C::EW);
    mbar_init(BAR(C::B_ACCFULL), 1);
    mbar_init(BAR(C::B_ACCEMPTY), C::EW);
    mbar_init(BAR(C::B_DRAIN), 1);
    mbar_init(BAR(C::B_DRAIN2), 1);
    mbar_init(BAR(C::B_DRAIN3), 1);
    misc[1] = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tmap(&p.tm_a);
    prefetch_tmap(&p.tm_b);
    prefetch_tmap(&p.tm_c);
    prefetch_tmap(&p.tm_d);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(misc))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  const int i_begin = p.cta_off[blockIdx.x], i_end = p.cta_off[blockIdx.x + 1];
  // job g's K tile in slot g % KST of the K ring, its V tile in slot KST + g % VST
  auto kslot = [](uint32_t g) { return g % C::KST; };
  auto vslot = [](uint32_t g) { return C::KST + g % C::VST; };
  auto tile = [&](uint32_t slot) { return sbase + C::OFF_RING + slot * C::TILE_BYTES; };

  if (warp == 0) {
    // ---- TMA producer: Q and dO once per item, then K and V tiles of every job (paged: one
    // lane per page); the whole warp runs the loop ----
    {
      uint32_t g = 0;
      int n = 0, a_last = -1;
      bool ok = true;
      for (int ii = i_begin; ok && ii < i_end; ++ii, ++n) {
        const BwdItem it = p.items[p.cta_items[ii]];
        if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_AEMPTY), (n & 1) ^ 1, guard, kBwdWaitAEmpty))) break;
        if (!((p.debug_flags & 1) && n == 0)) {
          a_last = n;
          if (lane == 0) mbar_expect_tx(BAR(C::B_AFULL), 2 * C::TILE_BYTES);
          __syncwarp();   // the expected byte count is posted before the copies
          if (lane < 2 * C::NBOX) {   // one box per lane: one issuing thread caps the copy rate
            const int c = lane % C::NBOX;
            tma_load_3d(sbase + (lane < C::NBOX ? C::OFF_A : C::OFF_B) + c * C::BOX_BYTES,
                        lane < C::NBOX ? &p.tm_a : &p.tm_b, c * 64, it.head, it.tok, BAR(C::B_AFULL));
          }
        }
        for (int j = 0; ok && j < it.job_count; ++j, ++g) {
          const BwdJob jb = p.jobs[it.job_start + j];
          for (int op = 0; op < 2; ++op) {
            const uint32_t slot = op == 0 ? kslot(g) : vslot(g), use = op == 0 ? g / C::KST : g / C::VST;
            if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_REMPTY + slot), (use & 1) ^ 1, guard, kBwdWaitREmpty))) {
              ok = false;
              break;
            }
            const CUtensorMap* tm = op == 0 ? &p.tm_c : &p.tm_d;
            if (lane == 0) mbar_expect_tx(BAR(C::B_RFULL + slot), C::TILE_BYTES);
            __syncwarp();   // the expected byte count is posted before the copies
            if constexpr (C::PAGED) {
              load_paged_tile<C::NBOX>(p, tm, tile(slot), it.seq, jb.tok, it.npages, it.kv_head, BAR(C::B_RFULL + slot),
                                       lane);
            } else if (lane < C::NBOX) {
              tma_load_3d(tile(slot) + lane * C::BOX_BYTES, tm, lane * 64, it.kv_head, jb.tok, BAR(C::B_RFULL + slot));
            }
          }
        }
      }
      // let the loads in flight land before the CTA exits
      if (lane == 0) {
        for (uint32_t x = g > uint32_t(C::KST) ? g - C::KST : 0u; x < g; ++x)
          wait_drain(BAR(C::B_RFULL + kslot(x)), (x / C::KST) & 1, p.timeout_ns);
        for (uint32_t x = g > uint32_t(C::VST) ? g - C::VST : 0u; x < g; ++x)
          wait_drain(BAR(C::B_RFULL + vslot(x)), (x / C::VST) & 1, p.timeout_ns);
        if (a_last >= 0) wait_drain(BAR(C::B_AFULL), a_last & 1, p.timeout_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---- S issuer. Job g (counted over the CTA's items): S = Q K^T into S slot g % 2 once
    // the dQ MMA of job g - 2 has completed
    if (lane == 0) {
      uint32_t g = 0;
      int n = 0;
      bool ok = true;
      for (int ii = i_begin; ok && ii < i_end; ++ii, ++n) {
        const BwdItem it = p.items[p.cta_items[ii]];
        if (!wait_bounded(BAR(C::B_AFULL), n & 1, guard, kBwdWaitAFull)) break;
        for (int j = 0; ok && j < it.job_count; ++j, ++g) {
          const uint32_t s = g & 1, ks = kslot(g);
          ok = wait_bounded(BAR(C::B_SFREE + s), ((g >> 1) & 1) ^ 1, guard, kBwdWaitSFree) &&
               wait_bounded(BAR(C::B_RFULL + ks), (g / C::KST) & 1, guard, kBwdWaitRFull);
          if (!ok) break;
          tc_fence_after();
          if constexpr (C::PAGED) {
            const int kr = p.jobs[it.job_start + j].rows;
            if (kr < 128) zero_tile_rows<C::NBOX>(tile(ks), kr);
          }
          mma_tile_ss<C::D>(tmem + C::TM_S + 128 * s, sbase + C::OFF_A, tile(ks), C::IDESC_SS);   // S = Q K^T
          mma_commit(BAR(C::B_SFULL + s));
        }
        if (!ok) break;
        mma_commit(BAR(C::B_AEMPTY));   // Q is read by these MMAs only
      }
      mma_commit(BAR(C::B_DRAIN));
      wait_drain(BAR(C::B_DRAIN), 0, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp == 3) {
    // ---- dP issuer: dP = dO V^T of job g into the dP slot once the warpgroups have read dP
    // of job g - 1
    if (lane == 0) {
      uint32_t g = 0;
      int n = 0;
      bool ok = true;
      for (int ii = i_begin; ok && ii < i_end; ++ii, ++n) {
        const BwdItem it = p.items[p.cta_items[ii]];
        if (!wait_bounded(BAR(C::B_AFULL), n & 1, guard, kBwdWaitAFull)) break;
        for (int j = 0; ok && j < it.job_count; ++j, ++g) {
          const uint32_t vs = vslot(g);
          ok = wait_bounded(BAR(C::B_READ), (g & 1) ^ 1, guard, kBwdWaitDpRead) &&
               wait_bounded(BAR(C::B_RFULL + vs), (g / C::VST) & 1, guard, kBwdWaitRFull);
          if (!ok) break;
          tc_fence_after();
          if constexpr (C::PAGED) {
            const int kr = p.jobs[it.job_start + j].rows;
            if (kr < 128) zero_tile_rows<C::NBOX>(tile(vs), kr);
          }
          mma_tile_ss<C::D>(tmem + C::TM_P, sbase + C::OFF_B, tile(vs), C::IDESC_SS);   // dP = dO V^T
          mma_commit(BAR(C::B_DPFULL));
          mma_commit(BAR(C::B_REMPTY + vs));   // V is read by this MMA only
        }
        if (!ok) break;
        mma_commit(BAR(C::B_AEMPTY));   // dO is read by these MMAs only
      }
      mma_commit(BAR(C::B_DRAIN3));
      wait_drain(BAR(C::B_DRAIN3), 0, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ---- dQ issuer: dQ += dS K once the warpgroups have written dS over the job's S slot;
    // frees the slot and the K tile on completion
    if (lane == 0) {
      uint32_t g = 0;
      int n = 0;
      bool ok = true;
      for (int ii = i_begin; ok && ii < i_end; ++ii, ++n) {
        const BwdItem it = p.items[p.cta_items[ii]];
        for (int j = 0; ok && j < it.job_count; ++j, ++g) {
          const uint32_t s = g & 1, ks = kslot(g);
          ok = wait_bounded(BAR(C::B_DSREADY + s), (g >> 1) & 1, guard, kBwdWaitDsReady);
          if (ok && j == 0) ok = wait_bounded(BAR(C::B_ACCEMPTY), (n & 1) ^ 1, guard, kBwdWaitAccEmpty);
          if (!ok) break;
          tc_fence_after();
          mma_tile_ts(tmem + C::TM_ACC, tmem + C::TM_S + 128 * s, tile(ks), C::IDESC_TS, j > 0 ? 1u : 0u);
          mma_commit(BAR(C::B_SFREE + s));
          mma_commit(BAR(C::B_REMPTY + ks));
        }
        if (!ok) break;
        mma_commit(BAR(C::B_ACCFULL));
      }
      mma_commit(BAR(C::B_DRAIN2));
      wait_drain(BAR(C::B_DRAIN2), 0, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ---- two elementwise warpgroups: thread r of warpgroup w owns row r of the query tile
    // and keys 64 w .. 64 w + 63 of every job ----
    const int r = (warp & 3) * 32 + lane, w = (warp - 4) >> 2;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const float sl2 = p.scale_log2;
    uint32_t g = 0;
    int n = 0;
    bool ok = true;
    for (int ii = i_begin; ok && ii < i_end; ++ii, ++n) {
      const BwdItem it = p.items[p.cta_items[ii]];
      const bool valid = r < it.rows;
      const int64_t grow = int64_t(it.tok + r) * p.hq + it.head;
      float lse2 = INFINITY, dlt = 0.f;   // lse2 = +inf: the row contributes nothing
      if (valid) {
        const float l = p.lse[grow];
        lse2 = l == -INFINITY ? INFINITY : l * 1.4426950408889634f;
        dlt = p.delta[grow];
      }
      const uint64_t sl2x2 = pk2(sl2, sl2), nlse2x2 = pk2(-lse2, -lse2), ndlt2 = pk2(-dlt, -dlt);
      // mask bits one job ahead, mask tile indices two jobs ahead: no global load latency
      // between two jobs
      const int nj = it.job_count;
      int mi_next = nj > 1 ? p.jobs[it.job_start + 1].mask : kMaskNone;
      uint4 bits_next = row_bits(p.mask_tiles, p.jobs[it.job_start].mask, r);
      for (int j = 0; ok && j < nj; ++j, ++g) {
        const uint4 bits4 = bits_next;
        bits_next = row_bits(p.mask_tiles, mi_next, r);
        mi_next = j + 2 < nj ? p.jobs[it.job_start + j + 2].mask : kMaskNone;
        const uint32_t s = g & 1;
        if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_SFULL + s), (g >> 1) & 1, guard, kBwdWaitSFull) &&
                                         wait_bounded(BAR(C::B_DPFULL), g & 1, guard, kBwdWaitDpFull))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t ts = tmem + lane_base + C::TM_S + 128 * s + 64 * w;
        // this warpgroup's 64 dP columns, then the slot is free for the next job's dP
        uint32_t dv[64], sv[32];
        tmem_ld32x32(tmem + lane_base + C::TM_P + 64 * w, dv);
        tmem_ld32x32(tmem + lane_base + C::TM_P + 64 * w + 32, dv + 32);
        tmem_ld32x32(ts, sv);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(BAR(C::B_READ));
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          if (c == 1) {
            tmem_ld32x32(ts + 32, sv);
            tmem_wait_ld();
          }
          const uint32_t wb = w ? (c ? bits4.w : bits4.z) : (c ? bits4.y : bits4.x);   // keys 64 w + 32 c ..
          const uint32_t* d32 = dv + 32 * c;
          uint32_t pk[16];
          if (wb == 0xffffffffu) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              // packed pairs: x = s sl2 - lse2, ds = 2^x (dp - delta)
              const uint64_t x = ffma2(pk2(__uint_as_float(sv[2 * e]), __uint_as_float(sv[2 * e + 1])), sl2x2, nlse2x2);
              const uint64_t pr = exp2_pair(x);
              const uint64_t dd = fadd2(pk2(__uint_as_float(d32[2 * e]), __uint_as_float(d32[2 * e + 1])), ndlt2);
              pk[e] = pack_bf16x2(fmul2(pr, dd));
            }
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              float ds[2];
#pragma unroll
              for (int q = 0; q < 2; ++q) {
                const float pr =
                    ((wb >> (2 * e + q)) & 1u) ? ex2(fmaf(__uint_as_float(sv[2 * e + q]), sl2, -lse2)) : 0.f;
                ds[q] = pr * (__uint_as_float(d32[2 * e + q]) - dlt);
              }
              pk[e] = pack_bf16(ds[0], ds[1]);
            }
          }
          // dS (bf16 pairs) of keys 64 w + 32 c .. over S columns 64 w + 16 c .. (already read)
          tmem_st32x16(ts + 16 * c, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(BAR(C::B_DSREADY + s));
      }
      if (!ok) break;
      if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_ACCFULL), n & 1, guard, kBwdWaitAccFull))) break;
      tc_fence_after();
      // warpgroup w stores columns D/2 w .. D/2 w + D/2 - 1 of the row's dq
      store_grad_cols<C::D / 2>(tmem + lane_base + C::TM_ACC + (C::D / 2) * w, p.scale, valid,
                                p.g0 + grow * C::D + (C::D / 2) * w);
      tc_fence_before();
      mbar_arrive(BAR(C::B_ACCEMPTY));
    }
  }
#undef BAR
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
}

// ================================ dK / dV ================================
template <class C>
__global__ void __launch_bounds__(C::THREADS, 1) masked_attn_bwd_dkv_kernel(const __grid_constant__ BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw);
  uint32_t* misc = reinterpret_cast<uint32_t*>(sgen + C::OFF_MISC);
  const uint32_t bar0 = sbase + C::OFF_BAR;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Guard guard{smem_u32(misc + 1), 0u, p.status, p.timeout_ns};
#define BAR(i) (bar0 + 8u * uint32_t(i))
  if (tid == 0) {
    mbar_init(BAR(C::B_AFULL), 1);
    mbar_init(BAR(C::B_AEMPTY), 2);   // both S-side issuers commit
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(BAR(C::B_RFULL + s), 1);
      mbar_init(BAR(C::B_REMPTY + s), 1);
    }
    for (int b = 0; b < C::NS; ++b) {
      mbar_init(BAR(C::B_SFULL + b), 1);
      mbar_init(BAR(C::B_DPFULL + b), 1);
      mbar_init(BAR(C::B_READ + b), C::EW);
      mbar_init(BAR(C::B_DSREADY + b), C::EW);
      mbar_init(BAR(C::B_SFREE + b), 1);
    }
    mbar_init(BAR(C::B_ACCFULL), 1);
    mbar_init(BAR(C::B_ACCEMPTY), C::EW);
    mbar_init(BAR(C::B_DRAIN), 1);
    mbar_init(BAR(C::B_DRAIN2), 1);
    mbar_init(BAR(C::B_DRAIN3), 1);
    misc[1] = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tmap(&p.tm_a);
    prefetch_tmap(&p.tm_b);
    prefetch_tmap(&p.tm_c);
    prefetch_tmap(&p.tm_d);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(misc))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  const int i_begin = p.cta_off[blockIdx.x], i_end = p.cta_off[blockIdx.x + 1];
  auto ring = [&](uint32_t r) { return sbase + C::OFF_RING + (r % C::STAGES) * C::TILE_BYTES; };

  if (warp == 0) {
    // ---- TMA producer: K and V once per item (paged: one lane per page), then Q and dO
    // tiles of every job; the whole warp runs the loop ----
    {
      uint32_t rc = 0;
      int n = 0, a_last = -1;
      bool ok = true;
      for (int ii = i_begin; ok && ii < i_end; ++ii, ++n) {
        const BwdItem it = p.items[p.cta_items[ii]];
        if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_AEMPTY), (n & 1) ^ 1, guard, kBwdWaitAEmpty))) break;
        if (!((p.debug_flags & 1) && n == 0)) {
          a_last = n;
          if (lane == 0) mbar_expect_tx(BAR(C::B_AFULL), 2 * C::TILE_BYTES);
          if constexpr (C::PAGED) {
            __syncwarp();   // the expected byte count is posted before the copies
            load_paged_tile<C::NBOX>(p, &p.tm_a, sbase + C::OFF_A, it.seq, it.tok, it.npages, it.kv_head,
                                     BAR(C::B_AFULL), lane);
            load_paged_tile<C::NBOX>(p, &p.tm_b, sbase + C::OFF_B, it.seq, it.tok, it.npages, it.kv_head,
                                     BAR(C::B_AFULL), lane);
          } else {
            __syncwarp();
            if (lane < 2 * C::NBOX) {   // one box per lane
              const int c = lane % C::NBOX;
              tma_load_3d(sbase + (lane < C::NBOX ? C::OFF_A : C::OFF_B) + c * C::BOX_BYTES,
                          lane < C::NBOX ? &p.tm_a : &p.tm_b, c * 64, it.kv_head, it.tok, BAR(C::B_AFULL));
            }
          }
        }
        for (int j = 0; ok && j < it.job_count; ++j) {
          const BwdJob jb = p.jobs[it.job_start + j];
          for (int op = 0; op < 2; ++op, ++rc) {
            const uint32_t slot = rc % C::STAGES;
            if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_REMPTY + slot), ((rc / C::STAGES) & 1) ^ 1, guard,
                                                      kBwdWaitREmpty))) {
              ok = false;
              break;
            }
            const CUtensorMap* tm = op == 0 ? &p.tm_c : &p.tm_d;
            if (lane == 0) mbar_expect_tx(BAR(C::B_RFULL + slot), C::TILE_BYTES);
            __syncwarp();
            if (lane < C::NBOX)   // one box per lane
              tma_load_3d(sbase + C::OFF_RING + slot * C::TILE_BYTES + lane * C::BOX_BYTES, tm, lane * 64, jb.head,
                          jb.tok, BAR(C::B_RFULL + slot));
          }
        }
      }
      if (lane == 0) {
        for (uint32_t r = rc > uint32_t(C::STAGES) ? rc - C::STAGES : 0u; r < rc; ++r)
          wait_drain(BAR(C::B_RFULL + r % C::STAGES), (r / C::STAGES) & 1, p.timeout_ns);
        if (a_last >= 0) wait_drain(BAR(C::B_AFULL), a_last & 1, p.timeout_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---- S^T issuer. Job g runs in TMEM slot g % 2: S^T = K Q^T once the dV and dK MMAs
    // of job g - 2 have completed
    if (lane == 0) {
      uint32_t rc = 0, g = 0;
      int n = 0;
      bool ok = true;
      for (int ii = i_begin; ok && ii < i_end; ++ii, ++n) {
        const BwdItem it = p.items[p.cta_items[ii]];
        if (!wait_bounded(BAR(C::B_AFULL), n & 1, guard, kBwdWaitAFull)) break;
        for (int j = 0; ok && j < it.job_count; ++j, ++g, rc += 2) {
          const uint32_t s = g & 1, rq = rc;
          ok = wait_bounded(BAR(C::B_SFREE + s), ((g >> 1) & 1) ^ 1, guard, kBwdWaitSFree) &&
               wait_bounded(BAR(C::B_RFULL + rq % C::STAGES), (rq / C::STAGES) & 1, guard, kBwdWaitRFull);
          if (!ok) break;
          tc_fence_after();
          mma_tile_ss<C::D>(tmem + C::TM_S + 128 * s, sbase + C::OFF_A, ring(rq), C::IDESC_SS);   // S^T = K Q^T
          mma_commit(BAR(C::B_SFULL + s));
        }
        if (!ok) break;
        mma_commit(BAR(C::B_AEMPTY));   // K is read by these MMAs only
      }
      mma_commit(BAR(C::B_DRAIN));
      wait_drain(BAR(C::B_DRAIN), 0, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp == 3) {
    // ---- dP^T issuer: dP^T = V dO^T of job g over S^T in slot g % 2 once the warpgroups have
    // read S^T
    if (lane == 0) {
      uint32_t rc = 0, g = 0;
      int n = 0;
      bool ok = true;
      for (int ii = i_begin; ok && ii < i_end; ++ii, ++n) {
        const BwdItem it = p.items[p.cta_items[ii]];
        if (!wait_bounded(BAR(C::B_AFULL), n & 1, guard, kBwdWaitAFull)) break;
        for (int j = 0; ok && j < it.job_count; ++j, ++g, rc += 2) {
          const uint32_t s = g & 1, rd = rc + 1;
          ok = wait_bounded(BAR(C::B_READ + s), (g >> 1) & 1, guard, kBwdWaitDpRead) &&
               wait_bounded(BAR(C::B_RFULL + rd % C::STAGES), (rd / C::STAGES) & 1, guard, kBwdWaitRFull);
          if (!ok) break;
          tc_fence_after();
          mma_tile_ss<C::D>(tmem + C::TM_S + 128 * s, sbase + C::OFF_B, ring(rd), C::IDESC_SS);   // dP^T = V dO^T
          mma_commit(BAR(C::B_DPFULL + s));
        }
        if (!ok) break;
        mma_commit(BAR(C::B_AEMPTY));   // V is read by these MMAs only
      }
      mma_commit(BAR(C::B_DRAIN3));
      wait_drain(BAR(C::B_DRAIN3), 0, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ---- dV / dK issuer: dV += P^T dO and dK += dS^T Q once the warpgroups have written P^T
    // and dS^T into the job's slot; frees the slot and the job's Q and dO tiles on completion
    if (lane == 0) {
      uint32_t rc = 0, g = 0;
      int n = 0;
      bool ok = true;
      for (int ii = i_begin; ok && ii < i_end; ++ii, ++n) {
        const BwdItem it = p.items[p.cta_items[ii]];
        for (int j = 0; ok && j < it.job_count; ++j, ++g, rc += 2) {
          const uint32_t s = g & 1, rq = rc, rd = rc + 1, acc = j > 0 ? 1u : 0u;
          ok = wait_bounded(BAR(C::B_DSREADY + s), (g >> 1) & 1, guard, kBwdWaitDsReady);
          if (ok && j == 0) ok = wait_bounded(BAR(C::B_ACCEMPTY), (n & 1) ^ 1, guard, kBwdWaitAccEmpty);
          if (!ok) break;
          tc_fence_after();
          const uint32_t slot = tmem + C::TM_S + 128 * s;
          mma_tile_ts(tmem + C::TM_ACC, slot, ring(rd), C::IDESC_TS, acc);               // dV += P^T dO
          mma_tile_ts(tmem + C::TM_ACC + C::D, slot + 32, ring(rq), C::IDESC_TS, acc);   // dK += dS^T Q
          mma_commit(BAR(C::B_SFREE + s));
          mma_commit(BAR(C::B_REMPTY + rq % C::STAGES));   // Q: read by S^T and dK
          mma_commit(BAR(C::B_REMPTY + rd % C::STAGES));   // dO: read by dP^T and dV
        }
        if (!ok) break;
        mma_commit(BAR(C::B_ACCFULL));
      }
      mma_commit(BAR(C::B_DRAIN2));
      wait_drain(BAR(C::B_DRAIN2), 0, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ---- two elementwise warpgroups: thread r of warpgroup w owns key row r of the key tile
    // and query rows 64 w .. 64 w + 63 of every job ----
    const int r = (warp & 3) * 32 + lane, w = (warp - 4) >> 2;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const float sl2 = p.scale_log2;
    const uint64_t sl2x2 = pk2(sl2, sl2);
    // this warp's copy of the job's per-query-row terms, -lse log2 e and -delta (no barrier
    // across warps)
    float* rl2 = reinterpret_cast<float*>(sgen + C::OFF_ROWV) + (warp - 4) * 256;
    float* rdl = rl2 + 128;
    uint32_t g = 0;
    int n = 0;
    bool ok = true;
    for (int ii = i_begin; ok && ii < i_end; ++ii, ++n) {
      const BwdItem it = p.items[p.cta_items[ii]];
      // The next job's lse / delta and mask bits are loaded while this job runs, the job
      // record two jobs ahead: only an item's first job waits for global memory.
      const int nj = it.job_count;
      const BwdJob none{0, kMaskNone, 0, 0};
      BwdJob jb_next = nj > 1 ? p.jobs[it.job_start + 1] : none;
      float nl[4], nd[4];
      auto load_terms = [&](const BwdJob& jb) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int qr = 4 * lane + q;
          nl[q] = -INFINITY;
          nd[q] = 0.f;
          if (qr < jb.rows) {
            const int64_t gi = int64_t(jb.tok + qr) * p.hq + jb.head;
            nl[q] = p.lse[gi];
            nd[q] = p.delta[gi];
          }
        }
      };
      uint4 bits_next;
      {
        const BwdJob j0 = p.jobs[it.job_start];
        load_terms(j0);
        bits_next = row_bits(p.mask_tiles, j0.mask, r);
      }
      for (int j = 0; ok && j < nj; ++j, ++g) {
        // the job's query rows' lse (log2 e scaled; -inf, no key, as +inf) and delta into this
        // warp's copy
        __syncwarp();   // the previous job's reads of rl2 / rdl are done
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          rl2[4 * lane + q] = nl[q] == -INFINITY ? -INFINITY : -(nl[q] * 1.4426950408889634f);   // -lse2
          rdl[4 * lane + q] = -nd[q];                                                             // -delta
        }
        __syncwarp();
        const uint4 bits = bits_next;
        load_terms(jb_next);
        bits_next = row_bits(p.mask_tiles, jb_next.mask, r);
        jb_next = j + 2 < nj ? p.jobs[it.job_start + j + 2] : none;

        // S^T of query rows 64 w .. 64 w + 63 into registers; then dP^T may overwrite it
        const uint32_t s = g & 1;
        if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_SFULL + s), (g >> 1) & 1, guard, kBwdWaitSFull))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t ts = tmem + lane_base + C::TM_S + 128 * s + 64 * w;
        float pr[64];
        {
          uint32_t sv[64];
          tmem_ld32x32(ts, sv);
          tmem_ld32x32(ts + 32, sv + 32);
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(BAR(C::B_READ + s));
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const uint32_t wb = w ? (c ? bits.w : bits.z) : (c ? bits.y : bits.x);
            const float4* l2v = reinterpret_cast<const float4*>(rl2 + 64 * w + 32 * c);
            if (wb == 0xffffffffu) {
#pragma unroll
              for (int f = 0; f < 8; ++f) {
                const float4 la = l2v[f];   // -lse2 of four query rows
                const uint32_t* s4 = sv + 32 * c + 4 * f;
                const uint64_t x01 = ffma2(pk2(__uint_as_float(s4[0]), __uint_as_float(s4[1])), sl2x2, pk2(la.x, la.y));
                const uint64_t x23 = ffma2(pk2(__uint_as_float(s4[2]), __uint_as_float(s4[3])), sl2x2, pk2(la.z, la.w));
                float* p4 = pr + 32 * c + 4 * f;
                unpk2(exp2_pair(x01), p4[0], p4[1]);
                unpk2(exp2_pair(x23), p4[2], p4[3]);
              }
            } else {
#pragma unroll
              for (int f = 0; f < 8; ++f) {
                const float4 la = l2v[f];
                const float lq[4] = {la.x, la.y, la.z, la.w};
#pragma unroll
                for (int q = 0; q < 4; ++q)
                  pr[32 * c + 4 * f + q] = ((wb >> (4 * f + q)) & 1u)
                                               ? ex2(fmaf(__uint_as_float(sv[32 * c + 4 * f + q]), sl2, lq[q]))
                                               : 0.f;
              }
            }
          }
        }
        // dS^T = P^T (dP^T - delta). This warpgroup's dP^T columns 64 w .. 64 w + 63 then take
        // P^T (bf16 pairs, columns 64 w .. 64 w + 31) and dS^T (64 w + 32 .. 64 w + 63); the
        // second half is read first, so every write lands on columns already read.
        if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_DPFULL + s), (g >> 1) & 1, guard, kBwdWaitDpFull))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t tp = ts;
#pragma unroll
        for (int c = 1; c >= 0; --c) {
          uint32_t dv[32];
          tmem_ld32x32(tp + 32 * c, dv);
          tmem_wait_ld();
          const float4* dlv = reinterpret_cast<const float4*>(rdl + 64 * w + 32 * c);
          uint32_t pk[16];
#pragma unroll
          for (int f = 0; f < 8; ++f) {
            const float4 da = dlv[f];   // -delta of four query rows
            const float* pp = pr + 32 * c + 4 * f;
            pk[2 * f] = pack_bf16x2(fmul2(pk2(pp[0], pp[1]),
                                          fadd2(pk2(__uint_as_float(dv[4 * f]), __uint_as_float(dv[4 * f + 1])),
                                                pk2(da.x, da.y))));
            pk[2 * f + 1] = pack_bf16x2(fmul2(pk2(pp[2], pp[3]),
                                              fadd2(pk2(__uint_as_float(dv[4 * f + 2]), __uint_as_float(dv[4 * f + 3])),
                                                    pk2(da.z, da.w))));
          }
          tmem_st32x16(tp + 32 + 16 * c, pk);
        }
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = pack_bf16(pr[32 * c + 2 * e], pr[32 * c + 2 * e + 1]);
          tmem_st32x16(tp + 16 * c, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(BAR(C::B_DSREADY + s));
      }
      if (!ok) break;
      if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_ACCFULL), n & 1, guard, kBwdWaitAccFull))) break;
      tc_fence_after();
      // warpgroup 0 stores the row's dv, warpgroup 1 its dk (paged: into the row's cache slot)
      bool valid = r < it.rows;
      int64_t krow = it.tok + r;
      if constexpr (C::PAGED) {
        const int key = it.tok + r;
        const int32_t page = valid ? __ldg(p.page_table + int64_t(it.seq) * p.maxp + key / p.page_size) : -1;
        valid = valid && page >= 0 && page < p.num_pages;
        krow = int64_t(page) * p.page_size + key % p.page_size;
      }
      const int64_t grow = krow * p.hkv + it.kv_head;
      if (w == 0) store_grad_cols<C::D>(tmem + lane_base + C::TM_ACC, 1.f, valid, p.g1 + grow * C::D);
      else store_grad_cols<C::D>(tmem + lane_base + C::TM_ACC + C::D, p.scale, valid, p.g0 + grow * C::D);
      tc_fence_before();
      mbar_arrive(BAR(C::B_ACCEMPTY));
    }
  }
#undef BAR
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
}

// ============================== head_dim 256 ==============================
// At d = 256 neither kernel's head_dim-128 structure fits: a 128-row tile of one head is
// 64 KiB, so two resident tiles (Q and dO, or K and V) take 128 KiB and the streamed
// operands are brought in as 32 KiB half-tiles (128 of the 256 columns) through a ring of
// three slots; and dV plus dK would take all 512 TMEM columns, so the dK/dV kernel runs
// twice, once per half of the head dimension (p.dhalf), accumulating dV and dK for those
// 128 columns and recomputing S^T and dP^T (K = 256 as two K = 128 halves) in each pass.
// One thread issues every MMA of a job in order: dP (dP^T), S (S^T), then the accumulating
// MMAs once the warpgroups have written dS (P^T and dS^T); the tensor pipe runs one
// thread's MMAs in issue order, so the next job's S / dP may overwrite the slots the
// previous job's accumulating MMAs read. TMEM: S (S^T) 0, dP (dP^T) 128, accumulators 256
// (dQ: 256 columns; dK/dV: dV 256, dK 384).
template <bool PAGED_ = false>
struct Bwd256Cfg {
  static constexpr int D = 256;
  static constexpr bool PAGED = PAGED_;   // K / V from a paged cache
  static constexpr int BOX_BYTES = 128 * 128;          // 128 rows x 64 columns
  static constexpr int TILE_BYTES = 4 * BOX_BYTES;     // resident 128 x 256 tile
  static constexpr int HALF_BYTES = 2 * BOX_BYTES;     // streamed 128 x 128 half-tile
  static constexpr int RSLOTS = 3;
  static constexpr int OFF_A = 0, OFF_B = TILE_BYTES, OFF_RING = 2 * TILE_BYTES;
  static constexpr int OFF_BAR = OFF_RING + RSLOTS * HALF_BYTES;
  static constexpr int B_AFULL = 0, B_AEMPTY = 1, B_RFULL = 2, B_REMPTY = B_RFULL + RSLOTS,
                       B_SFULL = B_REMPTY + RSLOTS, B_DPFULL = B_SFULL + 1, B_READY = B_DPFULL + 1,
                       B_PREADY = B_READY + 1,   // dK/dV: P^T written (dV may start before dS^T)
                       B_ACCFULL = B_PREADY + 1, B_ACCEMPTY = B_ACCFULL + 1, B_DRAIN = B_ACCEMPTY + 1,
                       NBAR = B_DRAIN + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;       // [0] TMEM base, [1] abort flag
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;   // + slack to align the base to 1 KiB
  static constexpr int THREADS = 384;
  static constexpr int EW = 256;
  static constexpr int TM_S = 0, TM_P = 128, TM_ACC = 256;
  static constexpr uint32_t IDESC_SS =  // M=128, N=128, bf16 x bf16 -> fp32, both K-major
      (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(128 >> 3) << 17) | (uint32_t(128 >> 4) << 24);
  static constexpr uint32_t IDESC_TS =  // M=128, N=128 (one half of the head dimension), A from TMEM
      (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | (uint32_t(128 >> 3) << 17) | (uint32_t(128 >> 4) << 24);
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// C[128 x 128] (+)= A . B^T over K = 256: A a resident tile (two 32 KiB halves), B two
// half-tiles in ring slots b0 (columns 0..127) and b1 (128..255).
__device__ __forceinline__ void mma_ss_k256(uint32_t d, uint32_t a_tile, uint32_t b0, uint32_t b1, uint32_t idesc) {
  mma_ss_x8_k128(d, desc_of(desc_lo(a_tile, 16)), desc_of(desc_lo(b0, 16)), idesc, 0u);
  mma_ss_x8_k128(d, desc_of(desc_lo(a_tile + Bwd256Cfg<>::HALF_BYTES, 16)), desc_of(desc_lo(b1, 16)), idesc, 1u);
}

// Producer for the d = 256 kernels, run by the whole warp (waits agreed with a vote): the
// two resident tiles once per item (tm_a, tm_b at the item's rows and head), then four
// half-tiles per job in the order `order` names (each entry: 0 / 1 = tm_c half 0 / 1,
// 2 / 3 = tm_d half 0 / 1) through the ring. Contiguous copies go one box per lane; K / V from
// a paged cache (the dK/dV kernel's resident tiles, the dQ kernel's half-tiles) one lane per
// page.
template <class C>
__device__ __forceinline__ void bwd256_produce(const BwdParams& p, uint32_t sbase, uint32_t bar0, const Guard& guard,
                                               int i_begin, int i_end, bool dkv, const int order[4], int lane) {
#define BAR(i) (bar0 + 8u * uint32_t(i))
  uint32_t rc = 0;
  int n = 0, a_last = -1;
  bool ok = true;
  for (int ii = i_begin; ok && ii < i_end; ++ii, ++n) {
    const BwdItem it = p.items[p.cta_items[ii]];
    const int a_head = dkv ? it.kv_head : it.head;
    if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_AEMPTY), (n & 1) ^ 1, guard, kBwdWaitAEmpty))) break;
    if (!((p.debug_flags & 1) && n == 0)) {
      a_last = n;
      if (lane == 0) mbar_expect_tx(BAR(C::B_AFULL), 2 * C::TILE_BYTES);
      __syncwarp();   // the expected byte count is posted before the copies
      if (C::PAGED && dkv) {
        load_paged_tile<4>(p, &p.tm_a, sbase + C::OFF_A, it.seq, it.tok, it.npages, it.kv_head, BAR(C::B_AFULL), lane);
        load_paged_tile<4>(p, &p.tm_b, sbase + C::OFF_B, it.seq, it.tok, it.npages, it.kv_head, BAR(C::B_AFULL), lane);
      } else if (lane < 8) {   // one box per lane
        const int c = lane & 3;
        tma_load_3d(sbase + (lane < 4 ? C::OFF_A : C::OFF_B) + c * C::BOX_BYTES, lane < 4 ? &p.tm_a : &p.tm_b, c * 64,
                    a_head, it.tok, BAR(C::B_AFULL));
      }
    }
    for (int j = 0; ok && j < it.job_count; ++j) {
      const BwdJob jb = p.jobs[it.job_start + j];
      const int head = dkv ? jb.head : it.kv_head;
      for (int q = 0; q < 4; ++q, ++rc) {
        const uint32_t slot = rc % C::RSLOTS;
        if (!__all_sync(0xffffffffu,
                        wait_bounded(BAR(C::B_REMPTY + slot), ((rc / C::RSLOTS) & 1) ^ 1, guard, kBwdWaitREmpty))) {
          ok = false;
          break;
        }
        if (lane == 0) mbar_expect_tx(BAR(C::B_RFULL + slot), C::HALF_BYTES);
        __syncwarp();
        const CUtensorMap* tm = order[q] < 2 ? &p.tm_c : &p.tm_d;
        const int col = (order[q] & 1) * 128;
        const uint32_t dst = sbase + C::OFF_RING + slot * C::HALF_BYTES;
        if (C::PAGED && !dkv) {
          const int ps = p.page_size;
          if (lane < 128 / ps) {   // lane = page of the key tile
            const int idx = jb.tok / ps + lane;
            const int32_t page = idx < it.npages ? __ldg(p.page_table + int64_t(it.seq) * p.maxp + idx) : -1;
            int32_t row = p.num_pages * ps;   // fully out of bounds: the box reads zeros
            if (page >= 0 && page < p.num_pages) row = page * ps;
            for (int c = 0; c < 2; ++c)
              tma_load_3d(dst + c * C::BOX_BYTES + lane * ps * 128, tm, col + c * 64, head, row, BAR(C::B_RFULL + slot));
          }
        } else if (lane < 2) {   // one box per lane
          tma_load_3d(dst + lane * C::BOX_BYTES, tm, col + lane * 64, head, jb.tok, BAR(C::B_RFULL + slot));
        }
      }
    }
  }
  if (lane == 0) {
    for (uint32_t r = rc > uint32_t(C::RSLOTS) ? rc - C::RSLOTS : 0u; r < rc; ++r)
      wait_drain(BAR(C::B_RFULL + r % C::RSLOTS), (r / C::RSLOTS) & 1, p.timeout_ns);
    if (a_last >= 0) wait_drain(BAR(C::B_AFULL), a_last & 1, p.timeout_ns);
  }
#undef BAR
}

template <class C>
__device__ __forceinline__ void bwd256_setup(uint32_t bar0, uint32_t* misc, const BwdParams& p, int tid) {
#define BAR(i) (bar0 + 8u * uint32_t(i))
  if (tid == 0) {
    mbar_init(BAR(C::B_AFULL), 1);
    mbar_init(BAR(C::B_AEMPTY), 1);
    for (int s = 0; s < C::RSLOTS; ++s) {
      mbar_init(BAR(C::B_RFULL + s), 1);
      mbar_init(BAR(C::B_REMPTY + s), 1);
    }
    mbar_init(BAR(C::B_SFULL), 1);
    mbar_init(BAR(C::B_DPFULL), 1);
    mbar_init(BAR(C::B_READY), C::EW);
    mbar_init(BAR(C::B_PREADY), C::EW);
    mbar_init(BAR(C::B_ACCFULL), 1);
    mbar_init(BAR(C::B_ACCEMPTY), C::EW);
    mbar_init(BAR(C::B_DRAIN), 1);
    misc[1] = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tmap(&p.tm_a);
    prefetch_tmap(&p.tm_b);
    prefetch_tmap(&p.tm_c);
    prefetch_tmap(&p.tm_d);
  }
#undef BAR
}

// dQ at d = 256. Per job the ring carries V half 0, V half 1, K half 0, K half 1.
template <class C>
__global__ void __launch_bounds__(C::THREADS, 1) masked_attn_bwd256_dq_kernel(const __grid_constant__ BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem_raw + (sbase - raw) + C::OFF_MISC);
  const uint32_t bar0 = sbase + C::OFF_BAR;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Guard guard{smem_u32(misc + 1), 0u, p.status, p.timeout_ns};
#define BAR(i) (bar0 + 8u * uint32_t(i))
  bwd256_setup<C>(bar0, misc, p, tid);
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(misc))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  const int i_begin = p.cta_off[blockIdx.x], i_end = p.cta_off[blockIdx.x + 1];
  auto ring = [&](uint32_t r) { return sbase + C::OFF_RING + (r % C::RSLOTS) * C::HALF_BYTES; };

  if (warp == 0) {
    // ---- TMA producer: Q and dO once per item; V halves, then K halves of every job ----
    const int order[4] = {2, 3, 0, 1};   // tm_c = K, tm_d = V
    bwd256_produce<C>(p, sbase, bar0, guard, i_begin, i_end, false, order, lane);
    __syncwarp();
  } else if (warp == 1) {
    // ---- MMA issuer: dP = dO V^T, S = Q K^T, then dQ += dS K for each job ----
    if (lane == 0) {
      uint32_t rc = 0, g = 0;
      int n = 0;
      bool ok = true;
      for (int ii = i_begin; ok && ii < i_end; ++ii, ++n) {
        const BwdItem it = p.items[p.cta_items[ii]];
        if (!wait_bounded(BAR(C::B_AFULL), n & 1, guard, kBwdWaitAFull)) break;
        for (int j = 0; ok && j < it.job_count; ++j, ++g, rc += 4) {
          const uint32_t rv0 = rc, rv1 = rc + 1, rk0 = rc + 2, rk1 = rc + 3;
          ok = wait_bounded(BAR(C::B_RFULL + rv0 % C::RSLOTS), (rv0 / C::RSLOTS) & 1, guard, kBwdWaitRFull) &&
               wait_bounded(BAR(C::B_RFULL + rv1 % C::RSLOTS), (rv1 / C::RSLOTS) & 1, guard, kBwdWaitRFull);
          if (!ok) break;
          tc_fence_after();
          const int kr = C::PAGED ? p.jobs[it.job_start + j].rows : 128;
          if (kr < 128) {   // a paged cache's stale rows past the sequence's last key
            zero_tile_rows<2>(ring(rv0), kr);
            zero_tile_rows<2>(ring(rv1), kr);
          }
          mma_ss_k256(tmem + C::TM_P, sbase + C::OFF_B, ring(rv0), ring(rv1), C::IDESC_SS);   // dP = dO V^T
          mma_commit(BAR(C::B_DPFULL));
          mma_commit(BAR(C::B_REMPTY + rv0 % C::RSLOTS));
          mma_commit(BAR(C::B_REMPTY + rv1 % C::RSLOTS));
          ok = wait_bounded(BAR(C::B_RFULL + rk0 % C::RSLOTS), (rk0 / C::RSLOTS) & 1, guard, kBwdWaitRFull) &&
               wait_bounded(BAR(C::B_RFULL + rk1 % C::RSLOTS), (rk1 / C::RSLOTS) & 1, guard, kBwdWaitRFull);
          if (!ok) break;
          tc_fence_after();
          if (kr < 128) {
            zero_tile_rows<2>(ring(rk0), kr);
            zero_tile_rows<2>(ring(rk1), kr);
          }
          mma_ss_k256(tmem + C::TM_S, sbase + C::OFF_A, ring(rk0), ring(rk1), C::IDESC_SS);   // S = Q K^T
          mma_commit(BAR(C::B_SFULL));
          ok = wait_bounded(BAR(C::B_READY), g & 1, guard, kBwdWaitDsReady);
          if (ok && j == 0) ok = wait_bounded(BAR(C::B_ACCEMPTY), (n & 1) ^ 1, guard, kBwdWaitAccEmpty);
          if (!ok) break;
          tc_fence_after();
          const uint32_t acc = j > 0 ? 1u : 0u;
          mma_tile_ts(tmem + C::TM_ACC, tmem + C::TM_S, ring(rk0), C::IDESC_TS, acc);         // dQ[:, 0:128]
          mma_tile_ts(tmem + C::TM_ACC + 128, tmem + C::TM_S, ring(rk1), C::IDESC_TS, acc);   // dQ[:, 128:256]
          mma_commit(BAR(C::B_REMPTY + rk0 % C::RSLOTS));
          mma_commit(BAR(C::B_REMPTY + rk1 % C::RSLOTS));
        }
        if (!ok) break;
        mma_commit(BAR(C::B_ACCFULL));
        mma_commit(BAR(C::B_AEMPTY));
      }
      mma_commit(BAR(C::B_DRAIN));
      wait_drain(BAR(C::B_DRAIN), 0, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ---- two elementwise warpgroups: thread r of warpgroup w owns row r of the query tile
    // and keys 64 w .. 64 w + 63 of every job ----
    const int r = (warp & 3) * 32 + lane, w = (warp - 4) >> 2;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const float sl2 = p.scale_log2;
    uint32_t g = 0;
    int n = 0;
    bool ok = true;
    for (int ii = i_begin; ok && ii < i_end; ++ii, ++n) {
      const BwdItem it = p.items[p.cta_items[ii]];
      const bool valid = r < it.rows;
      const int64_t grow = int64_t(it.tok + r) * p.hq + it.head;
      float lse2 = INFINITY, dlt = 0.f;
      if (valid) {
        const float l = p.lse[grow];
        lse2 = l == -INFINITY ? INFINITY : l * 1.4426950408889634f;
        dlt = p.delta[grow];
      }
      const uint64_t sl2x2 = pk2(sl2, sl2), nlse2x2 = pk2(-lse2, -lse2), ndlt2 = pk2(-dlt, -dlt);
      for (int j = 0; ok && j < it.job_count; ++j, ++g) {
        const uint4 bits4 = row_bits(p.mask_tiles, p.jobs[it.job_start + j].mask, r);
        if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_SFULL), g & 1, guard, kBwdWaitSFull) &&
                                         wait_bounded(BAR(C::B_DPFULL), g & 1, guard, kBwdWaitDpFull))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t ts = tmem + lane_base + C::TM_S + 64 * w;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t sv[32], dv[32];
          tmem_ld32x32(ts + 32 * c, sv);
          tmem_ld32x32(tmem + lane_base + C::TM_P + 64 * w + 32 * c, dv);
          tmem_wait_ld();
          const uint32_t wb = w ? (c ? bits4.w : bits4.z) : (c ? bits4.y : bits4.x);
          uint32_t pk[16];
          if (wb == 0xffffffffu) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const uint64_t x = ffma2(pk2(__uint_as_float(sv[2 * e]), __uint_as_float(sv[2 * e + 1])), sl2x2, nlse2x2);
              const uint64_t dd = fadd2(pk2(__uint_as_float(dv[2 * e]), __uint_as_float(dv[2 * e + 1])), ndlt2);
              pk[e] = pack_bf16x2(fmul2(exp2_pair(x), dd));
            }
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              float ds[2];
#pragma unroll
              for (int q = 0; q < 2; ++q) {
                const float pr =
                    ((wb >> (2 * e + q)) & 1u) ? ex2(fmaf(__uint_as_float(sv[2 * e + q]), sl2, -lse2)) : 0.f;
                ds[q] = pr * (__uint_as_float(dv[2 * e + q]) - dlt);
              }
              pk[e] = pack_bf16(ds[0], ds[1]);
            }
          }
          tmem_st32x16(ts + 16 * c, pk);   // over S columns this warpgroup has read
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(BAR(C::B_READY));
      }
      if (!ok) break;
      if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_ACCFULL), n & 1, guard, kBwdWaitAccFull))) break;
      tc_fence_after();
      store_grad_cols<128>(tmem + lane_base + C::TM_ACC + 128 * w, p.scale, valid, p.g0 + grow * C::D + 128 * w);
      tc_fence_before();
      mbar_arrive(BAR(C::B_ACCEMPTY));
    }
  }
#undef BAR
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
}

// dK / dV at d = 256 for head-dim half h = p.dhalf. Per job the ring carries Q half 1-h,
// Q half h, dO half 1-h, dO half h: the other halves are needed for S^T and dP^T only and
// their slots free first.
template <class C>
__global__ void __launch_bounds__(C::THREADS, 1) masked_attn_bwd256_dkv_kernel(const __grid_constant__ BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem_raw + (sbase - raw) + C::OFF_MISC);
  const uint32_t bar0 = sbase + C::OFF_BAR;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = p.dhalf;
  const Guard guard{smem_u32(misc + 1), 0u, p.status, p.timeout_ns};
#define BAR(i) (bar0 + 8u * uint32_t(i))
  bwd256_setup<C>(bar0, misc, p, tid);
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(misc))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  const int i_begin = p.cta_off[blockIdx.x], i_end = p.cta_off[blockIdx.x + 1];
  auto ring = [&](uint32_t r) { return sbase + C::OFF_RING + (r % C::RSLOTS) * C::HALF_BYTES; };

  if (warp == 0) {
    // ---- TMA producer: K and V once per item; Q and dO halves of every job ----
    const int order[4] = {1 - h, h, 2 + (1 - h), 2 + h};   // tm_c = Q, tm_d = dO
    bwd256_produce<C>(p, sbase, bar0, guard, i_begin, i_end, true, order, lane);
    __syncwarp();
  } else if (warp == 1) {
    // ---- MMA issuer: S^T = K Q^T, dP^T = V dO^T, then dV_h += P^T dO_h once the warpgroups
    // have written P^T (they then compute dS^T) and dK_h += dS^T Q_h ----
    if (lane == 0) {
      uint32_t rc = 0, g = 0;
      int n = 0;
      bool ok = true;
      for (int ii = i_begin; ok && ii < i_end; ++ii, ++n) {
        const BwdItem it = p.items[p.cta_items[ii]];
        if (!wait_bounded(BAR(C::B_AFULL), n & 1, guard, kBwdWaitAFull)) break;
        for (int j = 0; ok && j < it.job_count; ++j, ++g, rc += 4) {
          // ring positions of Q half 0 / 1 and dO half 0 / 1 (half 1-h comes first)
          const uint32_t rq[2] = {rc + uint32_t(h == 0 ? 1 : 0), rc + uint32_t(h == 0 ? 0 : 1)};
          const uint32_t rd[2] = {rc + 2 + uint32_t(h == 0 ? 1 : 0), rc + 2 + uint32_t(h == 0 ? 0 : 1)};
          ok = wait_bounded(BAR(C::B_RFULL + rc % C::RSLOTS), (rc / C::RSLOTS) & 1, guard, kBwdWaitRFull) &&
               wait_bounded(BAR(C::B_RFULL + (rc + 1) % C::RSLOTS), ((rc + 1) / C::RSLOTS) & 1, guard, kBwdWaitRFull);
          if (!ok) break;
          tc_fence_after();
          mma_ss_k256(tmem + C::TM_S, sbase + C::OFF_A, ring(rq[0]), ring(rq[1]), C::IDESC_SS);   // S^T = K Q^T
          mma_commit(BAR(C::B_SFULL));
          mma_commit(BAR(C::B_REMPTY + rc % C::RSLOTS));   // Q half 1-h: read by S^T only
          ok = wait_bounded(BAR(C::B_RFULL + (rc + 2) % C::RSLOTS), ((rc + 2) / C::RSLOTS) & 1, guard, kBwdWaitRFull) &&
               wait_bounded(BAR(C::B_RFULL + (rc + 3) % C::RSLOTS), ((rc + 3) / C::RSLOTS) & 1, guard, kBwdWaitRFull);
          if (!ok) break;
          tc_fence_after();
          mma_ss_k256(tmem + C::TM_P, sbase + C::OFF_B, ring(rd[0]), ring(rd[1]), C::IDESC_SS);   // dP^T = V dO^T
          mma_commit(BAR(C::B_DPFULL));
          mma_commit(BAR(C::B_REMPTY + (rc + 2) % C::RSLOTS));   // dO half 1-h: read by dP^T only
          ok = wait_bounded(BAR(C::B_PREADY), g & 1, guard, kBwdWaitPFull);
          if (ok && j == 0) ok = wait_bounded(BAR(C::B_ACCEMPTY), (n & 1) ^ 1, guard, kBwdWaitAccEmpty);
          if (!ok) break;
          tc_fence_after();
          const uint32_t acc = j > 0 ? 1u : 0u;
          mma_tile_ts(tmem + C::TM_ACC, tmem + C::TM_S, ring(rc + 3), C::IDESC_TS, acc);   // dV_h += P^T dO_h
          mma_commit(BAR(C::B_REMPTY + (rc + 3) % C::RSLOTS));                            // dO half h
          ok = wait_bounded(BAR(C::B_READY), g & 1, guard, kBwdWaitDsReady);
          if (!ok) break;
          tc_fence_after();
          mma_tile_ts(tmem + C::TM_ACC + 128, tmem + C::TM_P, ring(rc + 1), C::IDESC_TS, acc);   // dK_h += dS^T Q_h
          mma_commit(BAR(C::B_REMPTY + (rc + 1) % C::RSLOTS));                                  // Q half h
        }
        if (!ok) break;
        mma_commit(BAR(C::B_ACCFULL));
        mma_commit(BAR(C::B_AEMPTY));
      }
      mma_commit(BAR(C::B_DRAIN));
      wait_drain(BAR(C::B_DRAIN), 0, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ---- two elementwise warpgroups: thread r of warpgroup w owns key row r of the key tile
    // and query rows 64 w .. 64 w + 63 of every job; lane i of a warp fetches the lse and
    // delta of the chunk's query row i and the warp shares them by shuffles ----
    const int r = (warp & 3) * 32 + lane, w = (warp - 4) >> 2;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const float sl2 = p.scale_log2;
    uint32_t g = 0;
    int n = 0;
    bool ok = true;
    for (int ii = i_begin; ok && ii < i_end; ++ii, ++n) {
      const BwdItem it = p.items[p.cta_items[ii]];
      for (int j = 0; ok && j < it.job_count; ++j, ++g) {
        const BwdJob jb = p.jobs[it.job_start + j];
        const uint4 bits = row_bits(p.mask_tiles, jb.mask, r);
        float l2c[2], dlc[2];   // -lse log2 e and -delta of this lane's query row of chunk 0 / 1
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int qr = 64 * w + 32 * c + lane;
          l2c[c] = -INFINITY;
          dlc[c] = 0.f;
          if (qr < jb.rows) {
            const int64_t gi = int64_t(jb.tok + qr) * p.hq + jb.head;
            const float l = p.lse[gi];
            l2c[c] = l == -INFINITY ? -INFINITY : -(l * 1.4426950408889634f);
            dlc[c] = -p.delta[gi];
          }
        }
        if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_SFULL), g & 1, guard, kBwdWaitSFull))) {
          ok = false;
          break;
        }
        tc_fence_after();
        // P^T of query rows 64 w .. 64 w + 63 (kept for dS^T), bf16 pairs over S^T columns
        // this warpgroup has read
        const uint32_t ts = tmem + lane_base + C::TM_S + 64 * w;
        float pr[64];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t sv[32];
          tmem_ld32x32(ts + 32 * c, sv);
          tmem_wait_ld();
          const uint32_t wb = w ? (c ? bits.w : bits.z) : (c ? bits.y : bits.x);
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float l2 = __shfl_sync(0xffffffffu, l2c[c], e);
            pr[32 * c + e] = ((wb >> e) & 1u) ? ex2(fmaf(__uint_as_float(sv[e]), sl2, l2)) : 0.f;
          }
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = pack_bf16(pr[32 * c + 2 * e], pr[32 * c + 2 * e + 1]);
          tmem_st32x16(ts + 16 * c, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(BAR(C::B_PREADY));   // dV_h += P^T dO_h may run while dS^T is computed
        if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_DPFULL), g & 1, guard, kBwdWaitDpFull))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t tp = tmem + lane_base + C::TM_P + 64 * w;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t dv[32];
          tmem_ld32x32(tp + 32 * c, dv);
          tmem_wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float d0 = __shfl_sync(0xffffffffu, dlc[c], 2 * e), d1 = __shfl_sync(0xffffffffu, dlc[c], 2 * e + 1);
            pk[e] = pack_bf16x2(fmul2(pk2(pr[32 * c + 2 * e], pr[32 * c + 2 * e + 1]),
                                      fadd2(pk2(__uint_as_float(dv[2 * e]), __uint_as_float(dv[2 * e + 1])),
                                            pk2(d0, d1))));
          }
          tmem_st32x16(tp + 16 * c, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(BAR(C::B_READY));
      }
      if (!ok) break;
      if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_ACCFULL), n & 1, guard, kBwdWaitAccFull))) break;
      tc_fence_after();
      // warpgroup 0 stores columns 128 h .. 128 h + 127 of the row's dv, warpgroup 1 of its dk
      // (paged: into the key's cache slot)
      bool valid = r < it.rows;
      int64_t krow = it.tok + r;
      if constexpr (C::PAGED) {
        const int key = it.tok + r;
        const int32_t page = valid ? __ldg(p.page_table + int64_t(it.seq) * p.maxp + key / p.page_size) : -1;
        valid = valid && page >= 0 && page < p.num_pages;
        krow = int64_t(page) * p.page_size + key % p.page_size;
      }
      const int64_t grow = krow * p.hkv + it.kv_head;
      if (w == 0) store_grad_cols<128>(tmem + lane_base + C::TM_ACC, 1.f, valid, p.g1 + grow * C::D + 128 * h);
      else store_grad_cols<128>(tmem + lane_base + C::TM_ACC + 128, p.scale, valid, p.g0 + grow * C::D + 128 * h);
      tc_fence_before();
      mbar_arrive(BAR(C::B_ACCEMPTY));
    }
  }
#undef BAR
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
}

template <class C>
attn_status_t launch_bwd(int ctas, const BwdParams& p, cudaStream_t stream) {
  if constexpr (C::DKV) {
    const cudaError_t attr = once_per_device([] {
      return cudaFuncSetAttribute(masked_attn_bwd_dkv_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  C::SMEM_BYTES);
    });
    if (attr != cudaSuccess) return ATTN_ERR_CUDA;
  } else {
    const cudaError_t attr = once_per_device([] {
      return cudaFuncSetAttribute(masked_attn_bwd_dq_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  C::SMEM_BYTES);
    });
    if (attr != cudaSuccess) return ATTN_ERR_CUDA;
  }
  if constexpr (C::DKV) masked_attn_bwd_dkv_kernel<C><<<ctas, C::THREADS, C::SMEM_BYTES, stream>>>(p);
  else masked_attn_bwd_dq_kernel<C><<<ctas, C::THREADS, C::SMEM_BYTES, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <bool DKV, bool PAGED>
attn_status_t launch_bwd256(int ctas, const BwdParams& p, cudaStream_t stream) {
  using C = Bwd256Cfg<PAGED>;
  if constexpr (DKV) {
    const cudaError_t attr = once_per_device([] {
      return cudaFuncSetAttribute(masked_attn_bwd256_dkv_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  C::SMEM_BYTES);
    });
    if (attr != cudaSuccess) return ATTN_ERR_CUDA;
    masked_attn_bwd256_dkv_kernel<C><<<ctas, C::THREADS, C::SMEM_BYTES, stream>>>(p);
  } else {
    const cudaError_t attr = once_per_device([] {
      return cudaFuncSetAttribute(masked_attn_bwd256_dq_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  C::SMEM_BYTES);
    });
    if (attr != cudaSuccess) return ATTN_ERR_CUDA;
    masked_attn_bwd256_dq_kernel<C><<<ctas, C::THREADS, C::SMEM_BYTES, stream>>>(p);
  }
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace
}  // namespace mfa

attn_status_t mfa_launch_backward(const attn_plan_t* plan, const void* q, const void* k, const void* v,
                                  const void* out, const float* lse, const void* dout, const float* dlse, void* dq,
                                  void* dk, void* dv, cudaStream_t stream) {
  using namespace mfa;
  const int D = plan->d;
  const int64_t qrows = plan->total_q * plan->hq, krows = plan->total_kv_rows * plan->hkv;
  if (plan->total_q == 0 || plan->total_kv_rows == 0) {
    // nothing to attend: every gradient is zero
    cudaError_t e = cudaMemsetAsync(dq, 0, size_t(qrows) * D * 2, stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(dk, 0, size_t(krows) * D * 2, stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(dv, 0, size_t(krows) * D * 2, stream);
    return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
  }
  {
    const auto* o16 = static_cast<const __nv_bfloat16*>(out);
    const auto* g16 = static_cast<const __nv_bfloat16*>(dout);
    if (D == 64) bwd_delta_kernel<64><<<8 * 148, 256, 0, stream>>>(o16, g16, dlse, plan->d_bdelta, qrows);
    else if (D == 128) bwd_delta_kernel<128><<<8 * 148, 256, 0, stream>>>(o16, g16, dlse, plan->d_bdelta, qrows);
    else bwd_delta_kernel<256><<<8 * 148, 256, 0, stream>>>(o16, g16, dlse, plan->d_bdelta, qrows);
  }
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  BwdParams pq{}, pk{};
  // paged: K / V boxes of one page; dk / dv cover the whole cache, and the rows no sequence
  // reads (other pages, the tail of a sequence's last page) stay zero
  const uint32_t kv_box = plan->paged ? uint32_t(plan->page_size) : 128u;
  if (!encode3d(&pq.tm_a, q, D, plan->hq, plan->total_q, 128) ||
      !encode3d(&pq.tm_b, dout, D, plan->hq, plan->total_q, 128) ||
      !encode3d(&pq.tm_c, k, D, plan->hkv, plan->total_kv_rows, kv_box) ||
      !encode3d(&pq.tm_d, v, D, plan->hkv, plan->total_kv_rows, kv_box))
    return ATTN_ERR_CUDA;
  if (plan->paged) {
    cudaError_t e = cudaMemsetAsync(dk, 0, size_t(krows) * D * 2, stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(dv, 0, size_t(krows) * D * 2, stream);
    if (e != cudaSuccess) return ATTN_ERR_CUDA;
  }
  pk.tm_a = pq.tm_c;   // K
  pk.tm_b = pq.tm_d;   // V
  pk.tm_c = pq.tm_a;   // Q
  pk.tm_d = pq.tm_b;   // dO
  for (BwdParams* p : {&pq, &pk}) {
    p->lse = lse;
    p->delta = plan->d_bdelta;
    p->status = plan->d_status;
    p->hq = plan->hq;
    p->hkv = plan->hkv;
    p->debug_flags = plan->debug_flags;
    p->scale = plan->scale;
    p->scale_log2 = plan->scale * 1.4426950408889634f;
    p->timeout_ns = plan->timeout_ns;
    p->page_table = plan->page_table;
    p->page_size = plan->page_size;
    p->num_pages = plan->num_pages;
    p->maxp = plan->max_pages;
  }
  pq.items = plan->d_bq_items;
  pq.jobs = plan->d_bq_jobs;
  pq.cta_off = plan->d_bq_cta_off;
  pq.cta_items = plan->d_bq_cta_items;
  pq.mask_tiles = plan->d_bmask_q;
  pq.g0 = static_cast<__nv_bfloat16*>(dq);
  pk.items = plan->d_bkv_items;
  pk.jobs = plan->d_bkv_jobs;
  pk.cta_off = plan->d_bkv_cta_off;
  pk.cta_items = plan->d_bkv_cta_items;
  pk.mask_tiles = plan->d_bmask_k;
  pk.g0 = static_cast<__nv_bfloat16*>(dk);
  pk.g1 = static_cast<__nv_bfloat16*>(dv);
  attn_status_t st;
  if (plan->paged && D == 64) {
    st = launch_bwd<BwdCfg<64, false, true>>(plan->bq_ctas, pq, stream);
    if (st == ATTN_OK) st = launch_bwd<BwdCfg<64, true, true>>(plan->bkv_ctas, pk, stream);
  } else if (plan->paged && D == 128) {
    st = launch_bwd<BwdCfg<128, false, true>>(plan->bq_ctas, pq, stream);
    if (st == ATTN_OK) st = launch_bwd<BwdCfg<128, true, true>>(plan->bkv_ctas, pk, stream);
  } else if (plan->paged) {
    st = launch_bwd256<false, true>(plan->bq_ctas, pq, stream);
    for (int h = 0; h < 2 && st == ATTN_OK; ++h) {
      pk.dhalf = h;
      st = launch_bwd256<true, true>(plan->bkv_ctas, pk, stream);
    }
  } else if (D == 64) {
    st = launch_bwd<BwdCfg<64, false>>(plan->bq_ctas, pq, stream);
    if (st == ATTN_OK) st = launch_bwd<BwdCfg<64, true>>(plan->bkv_ctas, pk, stream);
  } else if (D == 128) {
    st = launch_bwd<BwdCfg<128, false>>(plan->bq_ctas, pq, stream);
    if (st == ATTN_OK) st = launch_bwd<BwdCfg<128, true>>(plan->bkv_ctas, pk, stream);
  } else {
    st = launch_bwd256<false, false>(plan->bq_ctas, pq, stream);
    for (int h = 0; h < 2 && st == ATTN_OK; ++h) {
      pk.dhalf = h;
      st = launch_bwd256<true, false>(plan->bkv_ctas, pk, stream);
    }
  }
  return st;
}
