// Masked attention backward for sm_100a (B200): dQ, dK and dV of the forward in attn_fwd.cu.
//
// With p_ij = exp(scale q_i . k_j - lse_i) on visible pairs (0 elsewhere), dp_ij = dout_i . v_j,
// delta_i = dout_i . out_i and ds_ij = p_ij (dp_ij - delta_i):
//     dq_i = scale sum_j ds_ij k_j,   dk_j = scale sum_i ds_ij q_i,   dv_j = sum_i p_ij dout_i,
// dk and dv of a key/value head summed over the query heads that read it. Three kernels:
//   bwd_delta_kernel    delta_i for every (row, query head): one warp per row.
//   dQ kernel           one persistent CTA per SM over dQ items (a 128-row query tile of one
//                       query head and its non-empty key tiles): S = Q K^T and dP = dO V^T
//                       into TMEM, the elementwise warpgroup turns them into dS (bf16, written
//                       over S), then dQ += dS K accumulates in TMEM.
//   dK/dV kernel        one persistent CTA per SM over dK/dV items (a 128-key tile of one
//                       key/value head and every (query head, query tile) that sees it):
//                       S^T = K Q^T and dP^T = V dO^T into TMEM, the warpgroup writes P^T and
//                       dS^T (bf16) over them, then dV += P^T dO and dK += dS^T Q accumulate in
//                       TMEM.
// Both recompute P from the forward's lse instead of storing it. Warp roles as in the
// forward: warp 0 TMA producer, warp 1 MMA issuer (one thread), warps 4-7 the elementwise
// warpgroup, one TMEM lane (= one tile row) per thread. Tiles are 128 rows of one head,
// 64-column boxes with the 128-byte swizzle; a ring of STAGES tile slots streams the
// per-job operands (dQ: K and V tiles; dK/dV: Q and dO tiles). Each job runs as two half
// jobs of 64 columns (keys for dQ, query rows for dK/dV) with two S / dP slots in TMEM, so
// the S / dP MMAs of the next half job overlap the elementwise work on the current one.
// TMEM: S slots at columns 0 and 64, dP slots at 128 and 192, the accumulators from 256
// (dQ: D columns; dK/dV: dV then dK). Every mbarrier wait is bounded as in the forward.
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
  float scale, scale_log2;
  int64_t timeout_ns;
};

template <int D_>
struct BwdCfg {
  static constexpr int D = D_;
  static constexpr int NBOX = D / 64;                  // 64-column boxes per tile
  static constexpr int BOX_BYTES = 128 * 128;          // 128 rows x 128 bytes
  static constexpr int TILE_BYTES = NBOX * BOX_BYTES;  // one 128-row tile of one head
  static constexpr int STAGES = D == 128 ? 4 : 8;      // ring tile slots (two per job)
  static constexpr int OFF_A = 0, OFF_B = TILE_BYTES, OFF_RING = 2 * TILE_BYTES;
  static constexpr int OFF_ROWV = OFF_RING + STAGES * TILE_BYTES;  // dK/dV: per warp 128 lse2 + 128 delta
  static constexpr int OFF_BAR = OFF_ROWV + 4 * 2 * 128 * 4;
  static constexpr int B_AFULL = 0, B_AEMPTY = 1, B_RFULL = 2, B_REMPTY = B_RFULL + STAGES,
                       B_SFULL = B_REMPTY + STAGES, B_PFULL = B_SFULL + 2, B_ACCFULL = B_PFULL + 2,
                       B_ACCEMPTY = B_ACCFULL + 1, B_DRAIN = B_ACCEMPTY + 1, NBAR = B_DRAIN + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;       // [0] TMEM base, [1] abort flag
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;   // + slack to align the base to 1 KiB
  static constexpr int THREADS = 256;
  // TMEM: S half-job slots at 0 and 64, dP slots at 128 and 192, accumulators from 256
  static constexpr int TM_S = 0, TM_P = 128, TM_ACC = 256;
  static constexpr int HALF_BYTES = 64 * 128;  // 64 rows of every 64-column box (8 swizzle atoms)
  static constexpr uint32_t IDESC_SS =  // M=128, N=64 (a half job), bf16 x bf16 -> fp32, both K-major
      (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(64 >> 3) << 17) | (uint32_t(128 >> 4) << 24);
  static constexpr uint32_t IDESC_TS =  // M=128, N=D, A from TMEM, B MN-major
      (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | (uint32_t(D >> 3) << 17) | (uint32_t(128 >> 4) << 24);
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(TM_ACC + 2 * D <= 512, "TMEM budget");
};

enum : int32_t {
  kBwdWaitAEmpty = 0x200, kBwdWaitREmpty, kBwdWaitAFull, kBwdWaitRFull, kBwdWaitPFull, kBwdWaitAccEmpty,
  kBwdWaitSFull, kBwdWaitAccFull
};

// C[128 x 64] (TMEM, fp32) = A[128 x D] . B[64 x D]^T: A a whole tile, B 64 rows of a tile
// (b_smem = tile + half * HALF_BYTES); both K-major in shared memory.
template <int D>
__device__ __forceinline__ void mma_half_ss(uint32_t d, uint32_t a_smem, uint32_t b_smem, uint32_t idesc) {
  if constexpr (D == 128) mma_ss_x8_k128(d, desc_of(desc_lo(a_smem, 16)), desc_of(desc_lo(b_smem, 16)), idesc, 0u);
  else mma_ss_x4_k64(d, desc_of(desc_lo(a_smem, 16)), desc_of(desc_lo(b_smem, 16)), idesc, 0u);
}

// C[128 x D] (+)= A[128 x 64] (bf16 in TMEM, 32 columns) . B[64 x D] (64 rows of a tile in
// shared memory, MN-major).
__device__ __forceinline__ void mma_half_ts(uint32_t d, uint32_t a_tmem, uint32_t b_smem, uint32_t idesc,
                                            uint32_t acc) {
  mma_ts_x4(d, a_tmem, desc_of(desc_lo(b_smem, 128 * 128)), idesc, acc);
}

// One 128-row x D tile of bf16 gradients from TMEM (fp32, times `mul`) to global memory.
template <int D>
__device__ __forceinline__ void store_grad_row(uint32_t t_acc, float mul, bool valid, __nv_bfloat16* dst) {
#pragma unroll 1
  for (int cc = 0; cc < D / 32; ++cc) {
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

// delta[r][h] = dout[r][h] . out[r][h] - dlse[r][h] (fp32; dlse may be null), one warp per
// (row, head). With a gradient on lse, ds = p (dp - delta) picks up + p dlse.
__global__ void bwd_delta_kernel(const __nv_bfloat16* __restrict__ out, const __nv_bfloat16* __restrict__ dout,
                                 const float* __restrict__ dlse, float* __restrict__ delta, int64_t rows, int D) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = int64_t(gridDim.x) * (blockDim.x >> 5);
  for (int64_t r = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
    float acc = 0.f;
    for (int c = 2 * lane; c < D; c += 64) {
      const __nv_bfloat162 o = *reinterpret_cast<const __nv_bfloat162*>(out + r * D + c);
      const __nv_bfloat162 g = *reinterpret_cast<const __nv_bfloat162*>(dout + r * D + c);
      acc = fmaf(__low2float(o), __low2float(g), acc);
      acc = fmaf(__high2float(o), __high2float(g), acc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) delta[r] = dlse ? acc - dlse[r] : acc;
  }
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
    mbar_init(BAR(C::B_AEMPTY), 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(BAR(C::B_RFULL + s), 1);
      mbar_init(BAR(C::B_REMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(BAR(C::B_SFULL + b), 1);
      mbar_init(BAR(C::B_PFULL + b), 128);
    }
    mbar_init(BAR(C::B_ACCFULL), 1);
    mbar_init(BAR(C::B_ACCEMPTY), 128);
    mbar_init(BAR(C::B_DRAIN), 1);
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

  if (warp == 0) {
    // ---- TMA producer: Q and dO once per item, then K and V tiles of every job ----
    if (lane == 0) {
      uint32_t rc = 0;
      int n = 0, a_last = -1;
      bool ok = true;
      for (int ii = i_begin; ok && ii < i_end; ++ii, ++n) {
        const BwdItem it = p.items[p.cta_items[ii]];
        if (!wait_bounded(BAR(C::B_AEMPTY), (n & 1) ^ 1, guard, kBwdWaitAEmpty)) break;
        if (!((p.debug_flags & 1) && n == 0)) {
          mbar_expect_tx(BAR(C::B_AFULL), 2 * C::TILE_BYTES);
          a_last = n;
          for (int c = 0; c < C::NBOX; ++c) {
            tma_load_3d(sbase + C::OFF_A + c * C::BOX_BYTES, &p.tm_a, c * 64, it.head, it.tok, BAR(C::B_AFULL));
            tma_load_3d(sbase + C::OFF_B + c * C::BOX_BYTES, &p.tm_b, c * 64, it.head, it.tok, BAR(C::B_AFULL));
          }
        }
        for (int j = 0; ok && j < it.job_count; ++j) {
          const BwdJob jb = p.jobs[it.job_start + j];
          for (int op = 0; op < 2; ++op, ++rc) {
            const uint32_t slot = rc % C::STAGES;
            if (!wait_bounded(BAR(C::B_REMPTY + slot), ((rc / C::STAGES) & 1) ^ 1, guard, kBwdWaitREmpty)) {
              ok = false;
              break;
            }
            mbar_expect_tx(BAR(C::B_RFULL + slot), C::TILE_BYTES);
            const CUtensorMap* tm = op == 0 ? &p.tm_c : &p.tm_d;
            for (int c = 0; c < C::NBOX; ++c)
              tma_load_3d(sbase + C::OFF_RING + slot * C::TILE_BYTES + c * C::BOX_BYTES, tm, c * 64, it.kv_head,
                          jb.tok, BAR(C::B_RFULL + slot));
          }
        }
      }
      for (uint32_t r = rc > uint32_t(C::STAGES) ? rc - C::STAGES : 0u; r < rc; ++r)
        wait_drain(BAR(C::B_RFULL + r % C::STAGES), (r / C::STAGES) & 1, p.timeout_ns);
      if (a_last >= 0) wait_drain(BAR(C::B_AFULL), a_last & 1, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---- MMA issuer: half jobs u = 2 j + h (keys 64 h .. 64 h + 63 of job j's tiles) ----
    // issued S(0), dP(0), S(1), dP(1), then dQ(u), S(u + 2), dP(u + 2): the MMAs of the next
    // half job run while the warpgroup works on the current one (two S / dP slots).
    if (lane == 0) {
      uint32_t rc = 0, gu = 0;
      int n = 0;
      bool ok = true;
      for (int ii = i_begin; ok && ii < i_end; ++ii, ++n) {
        const BwdItem it = p.items[p.cta_items[ii]];
        if (!wait_bounded(BAR(C::B_AFULL), n & 1, guard, kBwdWaitAFull)) break;
        tc_fence_after();
        const uint32_t base = rc;   // job j: K tile at ring index base + 2 j, V tile at base + 2 j + 1
        rc += 2 * uint32_t(it.job_count);
        const int U = 2 * it.job_count;
        auto ring = [&](uint32_t r) { return sbase + C::OFF_RING + (r % C::STAGES) * C::TILE_BYTES; };
        auto ss = [&](int u) -> bool {
          const uint32_t slot = (gu + u) & 1, rk = base + 2 * (u >> 1), rv = rk + 1, h = u & 1;
          if (h == 0) {
            if (!wait_bounded(BAR(C::B_RFULL + rk % C::STAGES), (rk / C::STAGES) & 1, guard, kBwdWaitRFull) ||
                !wait_bounded(BAR(C::B_RFULL + rv % C::STAGES), (rv / C::STAGES) & 1, guard, kBwdWaitRFull))
              return false;
            tc_fence_after();
          }
          mma_half_ss<C::D>(tmem + C::TM_S + 64 * slot, sbase + C::OFF_A, ring(rk) + h * C::HALF_BYTES,
                            C::IDESC_SS);   // S = Q K^T
          mma_half_ss<C::D>(tmem + C::TM_P + 64 * slot, sbase + C::OFF_B, ring(rv) + h * C::HALF_BYTES,
                            C::IDESC_SS);   // dP = dO V^T
          if (h == 1) mma_commit(BAR(C::B_REMPTY + rv % C::STAGES));
          mma_commit(BAR(C::B_SFULL + slot));
          return true;
        };
        auto ts = [&](int u) -> bool {
          const uint32_t g = gu + u, slot = g & 1, rk = base + 2 * (u >> 1), h = u & 1;
          if (!wait_bounded(BAR(C::B_PFULL + slot), (g >> 1) & 1, guard, kBwdWaitPFull)) return false;
          if (u == 0 && !wait_bounded(BAR(C::B_ACCEMPTY), (n & 1) ^ 1, guard, kBwdWaitAccEmpty)) return false;
          tc_fence_after();
          mma_half_ts(tmem + C::TM_ACC, tmem + C::TM_S + 64 * slot, ring(rk) + h * C::HALF_BYTES, C::IDESC_TS,
                      u > 0 ? 1u : 0u);     // dQ += dS K
          if (h == 1) mma_commit(BAR(C::B_REMPTY + rk % C::STAGES));
          return true;
        };
        ok = ss(0) && ss(1);
        for (int u = 0; ok && u < U; ++u) {
          ok = ts(u);
          if (ok && u + 2 < U) ok = ss(u + 2);
        }
        if (!ok) break;
        mma_commit(BAR(C::B_ACCFULL));
        mma_commit(BAR(C::B_AEMPTY));
        gu += U;
      }
      mma_commit(BAR(C::B_DRAIN));
      wait_drain(BAR(C::B_DRAIN), 0, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ---- elementwise warpgroup: thread r owns row r of the query tile ----
    const int r = tid - 128;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const float sl2 = p.scale_log2;
    uint32_t gu = 0;
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
      for (int u = 0; ok && u < 2 * it.job_count; ++u) {
        const int mi = p.jobs[it.job_start + (u >> 1)].mask;
        const int h = u & 1;
        uint2 bits = make_uint2(0xffffffffu, 0xffffffffu);   // this half job's 64 key bits
        if (mi >= 0) {
          const uint4 b4 = __ldg(p.mask_tiles + int64_t(mi) * 128 + r);
          bits = h ? make_uint2(b4.z, b4.w) : make_uint2(b4.x, b4.y);
        } else if (mi == kMaskNone) {
          bits = make_uint2(0u, 0u);
        }
        const uint32_t g = gu + u, slot = g & 1;
        if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_SFULL + slot), (g >> 1) & 1, guard, kBwdWaitSFull))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t sv[32], dv[32];
          tmem_ld32x32(tmem + lane_base + C::TM_S + 64 * slot + 32 * c, sv);
          tmem_ld32x32(tmem + lane_base + C::TM_P + 64 * slot + 32 * c, dv);
          tmem_wait_ld();
          const uint32_t w = c ? bits.y : bits.x;
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float ds[2];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const float pr = ((w >> (2 * e + q)) & 1u) ? ex2(fmaf(__uint_as_float(sv[2 * e + q]), sl2, -lse2)) : 0.f;
              ds[q] = pr * (__uint_as_float(dv[2 * e + q]) - dlt);
            }
            pk[e] = pack_bf16(ds[0], ds[1]);
          }
          // dS of the slot's columns 32c .. 32c+31 over its S columns 16c .. 16c+15 (already read)
          tmem_st32x16(tmem + lane_base + C::TM_S + 64 * slot + 16 * c, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(BAR(C::B_PFULL + slot));
      }
      gu += 2 * it.job_count;
      if (!ok) break;
      if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_ACCFULL), n & 1, guard, kBwdWaitAccFull))) break;
      tc_fence_after();
      store_grad_row<C::D>(tmem + lane_base + C::TM_ACC, p.scale, valid, p.g0 + grow * C::D);
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
    mbar_init(BAR(C::B_AEMPTY), 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(BAR(C::B_RFULL + s), 1);
      mbar_init(BAR(C::B_REMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(BAR(C::B_SFULL + b), 1);
      mbar_init(BAR(C::B_PFULL + b), 128);
    }
    mbar_init(BAR(C::B_ACCFULL), 1);
    mbar_init(BAR(C::B_ACCEMPTY), 128);
    mbar_init(BAR(C::B_DRAIN), 1);
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

  if (warp == 0) {
    // ---- TMA producer: K and V once per item, then Q and dO tiles of every job ----
    if (lane == 0) {
      uint32_t rc = 0;
      int n = 0, a_last = -1;
      bool ok = true;
      for (int ii = i_begin; ok && ii < i_end; ++ii, ++n) {
        const BwdItem it = p.items[p.cta_items[ii]];
        if (!wait_bounded(BAR(C::B_AEMPTY), (n & 1) ^ 1, guard, kBwdWaitAEmpty)) break;
        if (!((p.debug_flags & 1) && n == 0)) {
          mbar_expect_tx(BAR(C::B_AFULL), 2 * C::TILE_BYTES);
          a_last = n;
          for (int c = 0; c < C::NBOX; ++c) {
            tma_load_3d(sbase + C::OFF_A + c * C::BOX_BYTES, &p.tm_a, c * 64, it.kv_head, it.tok, BAR(C::B_AFULL));
            tma_load_3d(sbase + C::OFF_B + c * C::BOX_BYTES, &p.tm_b, c * 64, it.kv_head, it.tok, BAR(C::B_AFULL));
          }
        }
        for (int j = 0; ok && j < it.job_count; ++j) {
          const BwdJob jb = p.jobs[it.job_start + j];
          for (int op = 0; op < 2; ++op, ++rc) {
            const uint32_t slot = rc % C::STAGES;
            if (!wait_bounded(BAR(C::B_REMPTY + slot), ((rc / C::STAGES) & 1) ^ 1, guard, kBwdWaitREmpty)) {
              ok = false;
              break;
            }
            mbar_expect_tx(BAR(C::B_RFULL + slot), C::TILE_BYTES);
            const CUtensorMap* tm = op == 0 ? &p.tm_c : &p.tm_d;
            for (int c = 0; c < C::NBOX; ++c)
              tma_load_3d(sbase + C::OFF_RING + slot * C::TILE_BYTES + c * C::BOX_BYTES, tm, c * 64, jb.head, jb.tok,
                          BAR(C::B_RFULL + slot));
          }
        }
      }
      for (uint32_t r = rc > uint32_t(C::STAGES) ? rc - C::STAGES : 0u; r < rc; ++r)
        wait_drain(BAR(C::B_RFULL + r % C::STAGES), (r / C::STAGES) & 1, p.timeout_ns);
      if (a_last >= 0) wait_drain(BAR(C::B_AFULL), a_last & 1, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---- MMA issuer: half jobs u = 2 j + h (query rows 64 h .. 64 h + 63 of job j's tiles),
    // issued as in the dQ kernel: S^T(0), dP^T(0), S^T(1), dP^T(1), then dV, dK (u), S^T, dP^T (u + 2)
    if (lane == 0) {
      uint32_t rc = 0, gu = 0;
      int n = 0;
      bool ok = true;
      for (int ii = i_begin; ok && ii < i_end; ++ii, ++n) {
        const BwdItem it = p.items[p.cta_items[ii]];
        if (!wait_bounded(BAR(C::B_AFULL), n & 1, guard, kBwdWaitAFull)) break;
        tc_fence_after();
        const uint32_t base = rc;   // job j: Q tile at ring index base + 2 j, dO tile at base + 2 j + 1
        rc += 2 * uint32_t(it.job_count);
        const int U = 2 * it.job_count;
        auto ring = [&](uint32_t r) { return sbase + C::OFF_RING + (r % C::STAGES) * C::TILE_BYTES; };
        auto ss = [&](int u) -> bool {
          const uint32_t slot = (gu + u) & 1, rq = base + 2 * (u >> 1), rd = rq + 1, h = u & 1;
          if (h == 0) {
            if (!wait_bounded(BAR(C::B_RFULL + rq % C::STAGES), (rq / C::STAGES) & 1, guard, kBwdWaitRFull) ||
                !wait_bounded(BAR(C::B_RFULL + rd % C::STAGES), (rd / C::STAGES) & 1, guard, kBwdWaitRFull))
              return false;
            tc_fence_after();
          }
          mma_half_ss<C::D>(tmem + C::TM_S + 64 * slot, sbase + C::OFF_A, ring(rq) + h * C::HALF_BYTES,
                            C::IDESC_SS);   // S^T = K Q^T
          mma_half_ss<C::D>(tmem + C::TM_P + 64 * slot, sbase + C::OFF_B, ring(rd) + h * C::HALF_BYTES,
                            C::IDESC_SS);   // dP^T = V dO^T
          mma_commit(BAR(C::B_SFULL + slot));
          return true;
        };
        auto ts = [&](int u) -> bool {
          const uint32_t g = gu + u, slot = g & 1, rq = base + 2 * (u >> 1), rd = rq + 1, h = u & 1;
          if (!wait_bounded(BAR(C::B_PFULL + slot), (g >> 1) & 1, guard, kBwdWaitPFull)) return false;
          if (u == 0 && !wait_bounded(BAR(C::B_ACCEMPTY), (n & 1) ^ 1, guard, kBwdWaitAccEmpty)) return false;
          tc_fence_after();
          const uint32_t acc = u > 0 ? 1u : 0u;
          mma_half_ts(tmem + C::TM_ACC, tmem + C::TM_S + 64 * slot, ring(rd) + h * C::HALF_BYTES, C::IDESC_TS,
                      acc);                 // dV += P^T dO
          mma_half_ts(tmem + C::TM_ACC + C::D, tmem + C::TM_P + 64 * slot, ring(rq) + h * C::HALF_BYTES,
                      C::IDESC_TS, acc);    // dK += dS^T Q
          if (h == 1) {
            mma_commit(BAR(C::B_REMPTY + rq % C::STAGES));
            mma_commit(BAR(C::B_REMPTY + rd % C::STAGES));
          }
          return true;
        };
        ok = ss(0) && ss(1);
        for (int u = 0; ok && u < U; ++u) {
          ok = ts(u);
          if (ok && u + 2 < U) ok = ss(u + 2);
        }
        if (!ok) break;
        mma_commit(BAR(C::B_ACCFULL));
        mma_commit(BAR(C::B_AEMPTY));
        gu += U;
      }
      mma_commit(BAR(C::B_DRAIN));
      wait_drain(BAR(C::B_DRAIN), 0, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ---- elementwise warpgroup: thread r owns key row r of the key tile ----
    const int r = tid - 128;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const float sl2 = p.scale_log2;
    // this warp's copy of the job's per-query-row terms (no barrier across warps)
    float* rl2 = reinterpret_cast<float*>(sgen + C::OFF_ROWV) + (warp - 4) * 256;
    float* rdl = rl2 + 128;
    uint32_t gu = 0;
    int n = 0;
    bool ok = true;
    for (int ii = i_begin; ok && ii < i_end; ++ii, ++n) {
      const BwdItem it = p.items[p.cta_items[ii]];
      uint4 bits = make_uint4(0u, 0u, 0u, 0u);
      for (int u = 0; ok && u < 2 * it.job_count; ++u) {
        const int h = u & 1;
        if (h == 0) {
          // a new job: its query rows' lse (log2 e scaled) and delta into this warp's copy
          const BwdJob jb = p.jobs[it.job_start + (u >> 1)];
          __syncwarp();   // the previous job's reads of rl2 / rdl are done
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int qr = 4 * lane + k;
            float l2 = INFINITY, dl = 0.f;
            if (qr < jb.rows) {
              const int64_t g = int64_t(jb.tok + qr) * p.hq + jb.head;
              const float l = p.lse[g];
              l2 = l == -INFINITY ? INFINITY : l * 1.4426950408889634f;
              dl = p.delta[g];
            }
            rl2[qr] = l2;
            rdl[qr] = dl;
          }
          __syncwarp();
          bits = make_uint4(0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu);
          if (jb.mask >= 0) bits = __ldg(p.mask_tiles + int64_t(jb.mask) * 128 + r);
          else if (jb.mask == kMaskNone) bits = make_uint4(0u, 0u, 0u, 0u);
        }
        const uint32_t g = gu + u, slot = g & 1;
        if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_SFULL + slot), (g >> 1) & 1, guard, kBwdWaitSFull))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t sv[32], dv[32];
          tmem_ld32x32(tmem + lane_base + C::TM_S + 64 * slot + 32 * c, sv);
          tmem_ld32x32(tmem + lane_base + C::TM_P + 64 * slot + 32 * c, dv);
          tmem_wait_ld();
          const int q0 = 64 * h + 32 * c;   // first query row of the chunk
          const uint32_t w = h ? (c ? bits.w : bits.z) : (c ? bits.y : bits.x);
          uint32_t pp[16], pd[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float pr[2], ds[2];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const int qi = q0 + 2 * e + q;
              pr[q] = ((w >> (2 * e + q)) & 1u) ? ex2(fmaf(__uint_as_float(sv[2 * e + q]), sl2, -rl2[qi])) : 0.f;
              ds[q] = pr[q] * (__uint_as_float(dv[2 * e + q]) - rdl[qi]);
            }
            pp[e] = pack_bf16(pr[0], pr[1]);
            pd[e] = pack_bf16(ds[0], ds[1]);
          }
          // P^T over the slot's S^T columns 16c.., dS^T over its dP^T columns 16c.. (already read)
          tmem_st32x16(tmem + lane_base + C::TM_S + 64 * slot + 16 * c, pp);
          tmem_st32x16(tmem + lane_base + C::TM_P + 64 * slot + 16 * c, pd);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(BAR(C::B_PFULL + slot));
      }
      gu += 2 * it.job_count;
      if (!ok) break;
      if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_ACCFULL), n & 1, guard, kBwdWaitAccFull))) break;
      tc_fence_after();
      const bool valid = r < it.rows;
      const int64_t grow = int64_t(it.tok + r) * p.hkv + it.kv_head;
      store_grad_row<C::D>(tmem + lane_base + C::TM_ACC, 1.f, valid, p.g1 + grow * C::D);           // dv
      store_grad_row<C::D>(tmem + lane_base + C::TM_ACC + C::D, p.scale, valid, p.g0 + grow * C::D);  // dk
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

template <class C, bool DKV>
attn_status_t launch_bwd(int ctas, const BwdParams& p, cudaStream_t stream) {
  const cudaError_t attr = once_per_device([] {
    return DKV ? cudaFuncSetAttribute(masked_attn_bwd_dkv_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      C::SMEM_BYTES)
               : cudaFuncSetAttribute(masked_attn_bwd_dq_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      C::SMEM_BYTES);
  });
  if (attr != cudaSuccess) return ATTN_ERR_CUDA;
  if (DKV) masked_attn_bwd_dkv_kernel<C><<<ctas, C::THREADS, C::SMEM_BYTES, stream>>>(p);
  else masked_attn_bwd_dq_kernel<C><<<ctas, C::THREADS, C::SMEM_BYTES, stream>>>(p);
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
  bwd_delta_kernel<<<4 * 148, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(out),
                                                static_cast<const __nv_bfloat16*>(dout), dlse, plan->d_bdelta, qrows, D);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  BwdParams pq{}, pk{};
  if (!encode3d(&pq.tm_a, q, D, plan->hq, plan->total_q, 128) ||
      !encode3d(&pq.tm_b, dout, D, plan->hq, plan->total_q, 128) ||
      !encode3d(&pq.tm_c, k, D, plan->hkv, plan->total_kv_rows, 128) ||
      !encode3d(&pq.tm_d, v, D, plan->hkv, plan->total_kv_rows, 128))
    return ATTN_ERR_CUDA;
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
  if (D == 64) {
    st = launch_bwd<BwdCfg<64>, false>(plan->bq_ctas, pq, stream);
    if (st == ATTN_OK) st = launch_bwd<BwdCfg<64>, true>(plan->bkv_ctas, pk, stream);
  } else {
    st = launch_bwd<BwdCfg<128>, false>(plan->bq_ctas, pq, stream);
    if (st == ATTN_OK) st = launch_bwd<BwdCfg<128>, true>(plan->bkv_ctas, pk, stream);
  }
  return st;
}
