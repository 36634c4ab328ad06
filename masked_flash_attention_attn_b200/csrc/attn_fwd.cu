// Masked attention forward for sm_100a (B200).
//
// One persistent CTA per SM walks its list of work items (built by the planner). A work
// item is NQ 128-row query tiles (NQ = 2 for head_dim <= 128, 1 for head_dim 256) that
// share one key/value head and one run of key tiles; empty key tiles never appear in the
// run, full key tiles carry no mask, partial ones carry the index of a 2 KiB
// tile-transposed bit mask.
//
// Warp roles (128 * (1 + NQ) threads):
//   warp 0      TMA producer: Q tiles once per item, K and V tiles through a ring of
//               STAGES shared-memory chunks (128 keys x 128 columns, 128-byte swizzle);
//               paged K/V arrive as one box per page.
//   warp 1      MMA issuer (one thread): S = Q K^T into TMEM (tcgen05.mma, bf16 inputs,
//               fp32 accumulators) and O += P V with P read from TMEM.
//   warps 2-3   idle (they hold the warpgroup's TMEM lane quarters for the allocator).
//   warpgroup 1+t  softmax of query tile t: one thread per row reads its S row from TMEM
//               (tcgen05.ld), applies the row's 128 mask bits (one 16-byte load) on partial
//               tiles, keeps the online max / sum, writes P as bf16 back into the S
//               columns, rescales O in TMEM when the running max grows by more than 2^8,
//               and finally normalises O, writes out (bf16) and the row lse (fp32).
//
// The S accumulators are double buffered: the stream of (key tile, query tile) jobs of an
// item is issued as S(0), S(1), then P V(u), S(u + 2) for u = 0, 1, ..., so the tensor
// core works on the next job while the softmax warpgroup(s) work on the current one.
// TMEM (512 columns): S slot 0 at column 0, S slot 1 at 128, O of tile t at 256 + t D.
//
// Every wait on an mbarrier is bounded (globaltimer). When a wait expires the thread
// records ATTN_ERR_TIMEOUT in the plan's status word, raises a shared abort flag that
// ends every other wait, lets its own copies / MMAs in flight complete, and the CTA
// frees its TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "attn_internal.h"

namespace mfa {
namespace {

struct Params {
  CUtensorMap tm_q;
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  const WorkItem* items;
  const Job* jobs;
  const int32_t* cta_off;
  const int32_t* cta_items;
  const uint4* mask_tiles;
  const int32_t* page_table;
  __nv_bfloat16* out;
  float* lse;
  int32_t* status;
  int32_t hq, R, hp, page_size, num_pages, debug_flags;
  float scale_log2;
  int64_t timeout_ns;
};

template <int D_, int NQ_, int STAGES_, bool PAGED_>
struct Cfg {
  static constexpr int D = D_, NQ = NQ_, STAGES = STAGES_;
  static constexpr bool PAGED = PAGED_;
  static constexpr int CH = D < 128 ? D : 128;   // columns of one ring chunk
  static constexpr int NCH = D / CH;             // ring chunks per K or V tile
  static constexpr int NBOX = CH / 64;           // 64-column (128-byte) boxes per chunk
  static constexpr int QBOX = D / 64;            // 64-column boxes per Q tile
  static constexpr int BOX_BYTES = 128 * 128;    // 128 rows x 128 bytes
  static constexpr int Q_BYTES = QBOX * BOX_BYTES;
  static constexpr int CHUNK_BYTES = NBOX * BOX_BYTES;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_RING = NQ * Q_BYTES;
  static constexpr int OFF_BAR = OFF_RING + STAGES * CHUNK_BYTES;
  // mbarrier indices
  static constexpr int B_QFULL = 0, B_QEMPTY = 1, B_KVFULL = 2, B_KVEMPTY = B_KVFULL + STAGES,
                       B_SFULL = B_KVEMPTY + STAGES, B_PFULL = B_SFULL + 2, B_PVDONE = B_PFULL + 2,
                       B_OEMPTY = B_PVDONE + NQ, B_DRAIN = B_OEMPTY + NQ, NBAR = B_DRAIN + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;  // [0] TMEM base, [1] abort flag
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + slack to align the base to 1 KiB
  static constexpr int THREADS = 128 * (1 + NQ);
  static constexpr int TM_O = 256;
  static constexpr uint32_t IDESC_QK =  // M=128, N=128, bf16 x bf16 -> fp32, both K-major
      (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(128 >> 3) << 17) | (uint32_t(128 >> 4) << 24);
  static constexpr uint32_t IDESC_PV =  // M=128, N=CH, A (P) from TMEM K-major, B (V) MN-major
      (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | (uint32_t(CH >> 3) << 17) | (uint32_t(128 >> 4) << 24);
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(2 * 128 + NQ * D <= 512, "TMEM budget");
};

// ---- small PTX wrappers ------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t gtime() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint32_t ld_volatile_shared(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.volatile.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ void st_volatile_shared(uint32_t addr, uint32_t v) {
  asm volatile("st.volatile.shared.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

struct Guard {
  uint32_t abort_addr;
  int32_t* status;
  int64_t timeout_ns;
};

// Slow path of wait_bounded: spin on try_wait until the phase completes, the shared abort
// flag is raised (returns false) or timeout_ns passes (raises the flag, records `code`).
__device__ __noinline__ bool wait_slow(uint32_t bar, uint32_t parity, uint32_t abort_addr, int32_t* status,
                                       int64_t timeout_ns, int32_t code) {
  const uint64_t t0 = gtime();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 16; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (ld_volatile_shared(abort_addr) != 0u) return false;
    if (gtime() - t0 > uint64_t(timeout_ns)) {
      st_volatile_shared(abort_addr, 1u);
      atomicCAS(status, 0, code);
      return false;
    }
  }
}

// Wait for the phase of `parity` to complete; false when the CTA is aborting.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, const Guard& g, int32_t code) {
  if (mbar_try_wait(bar, parity)) return true;
  return wait_slow(bar, parity, g.abort_addr, g.status, g.timeout_ns, code);
}

// Wait without looking at the abort flag (used to let in-flight async work land before
// the CTA exits); still bounded.
__device__ __noinline__ void wait_drain(uint32_t bar, uint32_t parity, int64_t timeout_ns) {
  const uint64_t t0 = gtime();
  while (!mbar_try_wait(bar, parity)) {
    if (gtime() - t0 > uint64_t(timeout_ns)) return;
  }
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* tm, int32_t c0, int32_t c1, int32_t c2,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* tm) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tm)) : "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 version field = 1.
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return uint64_t((addr & 0x3FFFFu) >> 4) | (uint64_t(lbo >> 4) << 16) | (uint64_t(sbo >> 4) << 32) |
         (1ull << 46) | (2ull << 61);
}

__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

#include "tmem_ldst.inc"

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two fp32 -> one bf16x2 word (round to nearest even); `lo` lands in the low half, which
// is the lower column / key index in every layout used here.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// ---- the kernel ----------------------------------------------------------------------------

enum : int32_t {
  kWaitQEmpty = 0x100, kWaitKvEmpty, kWaitQFull, kWaitKvFull, kWaitPFull, kWaitOEmpty, kWaitSFull, kWaitPvDone
};

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1) masked_attn_fwd_kernel(const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem_raw + (sbase - raw) + C::OFF_MISC);
  const uint32_t bar0 = sbase + C::OFF_BAR;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Guard guard{smem_u32(misc + 1), p.status, p.timeout_ns};
#define BAR(i) (bar0 + 8u * uint32_t(i))

  if (tid == 0) {
    mbar_init(BAR(C::B_QFULL), 1);
    mbar_init(BAR(C::B_QEMPTY), 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(BAR(C::B_KVFULL + s), 1);
      mbar_init(BAR(C::B_KVEMPTY + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(BAR(C::B_SFULL + s), 1);
      mbar_init(BAR(C::B_PFULL + s), 128);
    }
    for (int t = 0; t < C::NQ; ++t) {
      mbar_init(BAR(C::B_PVDONE + t), 1);
      mbar_init(BAR(C::B_OEMPTY + t), 128);
    }
    mbar_init(BAR(C::B_DRAIN), 1);
    misc[1] = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tmap(&p.tm_q);
    prefetch_tmap(&p.tm_k);
    prefetch_tmap(&p.tm_v);
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
    // ================================ TMA producer ================================
    if (lane == 0) {
      uint32_t rc = 0;            // ring chunks issued
      int n = 0;
      int q_last = -1;            // last item whose Q load was armed
      for (int ii = i_begin; ii < i_end; ++ii, ++n) {
        const WorkItem it = p.items[p.cta_items[ii]];
        if (!wait_bounded(BAR(C::B_QEMPTY), (n & 1) ^ 1, guard, kWaitQEmpty)) break;
        if (!((p.debug_flags & 1) && n == 0)) {
          mbar_expect_tx(BAR(C::B_QFULL), C::NQ * C::Q_BYTES);
          q_last = n;
          for (int t = 0; t < C::NQ; ++t)
            for (int hh = 0; hh < p.hp; ++hh)
              for (int c = 0; c < C::QBOX; ++c)
                tma_load_3d(sbase + C::OFF_Q + t * C::Q_BYTES + c * C::BOX_BYTES + hh * p.R * 128, &p.tm_q, c * 64,
                            it.head[t] + hh, it.tok[t], BAR(C::B_QFULL));
        }
        const int T = C::NQ * it.job_count;
        auto load_tile = [&](bool is_v, int j) -> bool {
          const int kt = p.jobs[it.job_start + j].k_tile;
          const CUtensorMap* tm = is_v ? &p.tm_v : &p.tm_k;
          for (int h = 0; h < C::NCH; ++h, ++rc) {
            const uint32_t slot = rc % C::STAGES;
            if (!wait_bounded(BAR(C::B_KVEMPTY + slot), ((rc / C::STAGES) & 1) ^ 1, guard, kWaitKvEmpty))
              return false;
            mbar_expect_tx(BAR(C::B_KVFULL + slot), C::CHUNK_BYTES);
            const uint32_t dst = sbase + C::OFF_RING + slot * C::CHUNK_BYTES;
            if constexpr (!C::PAGED) {
              for (int c = 0; c < C::NBOX; ++c)
                tma_load_3d(dst + c * C::BOX_BYTES, tm, h * C::CH + c * 64, it.kv_head, it.k_base + kt * 128,
                            BAR(C::B_KVFULL + slot));
            } else {
              const int ps = p.page_size, ppt = 128 / ps;
              for (int pg = 0; pg < ppt; ++pg) {
                const int idx = kt * ppt + pg;
                int32_t row = p.num_pages * ps;  // fully out of bounds: the box reads zeros
                if (idx < it.npages) {
                  const int32_t page = __ldg(p.page_table + it.k_base + idx);
                  if (page >= 0 && page < p.num_pages) row = page * ps;
                }
                for (int c = 0; c < C::NBOX; ++c)
                  tma_load_3d(dst + c * C::BOX_BYTES + pg * ps * 128, tm, h * C::CH + c * 64, it.kv_head, row,
                              BAR(C::B_KVFULL + slot));
              }
            }
          }
          return true;
        };
        // loads in the order the MMA issuer consumes them
        bool ok = load_tile(false, 0);
        if (ok && T > 1 && C::NQ == 1) ok = load_tile(false, 1);
        for (int u = 0; ok && u < T; ++u) {
          if (u % C::NQ == 0) ok = load_tile(true, u / C::NQ);
          const int t = u + 2;
          if (ok && t < T && t % C::NQ == 0) ok = load_tile(false, t / C::NQ);
        }
        if (!ok) break;
      }
      // let every copy this thread issued land before the CTA may exit
      for (uint32_t r = rc > uint32_t(C::STAGES) ? rc - C::STAGES : 0u; r < rc; ++r)
        wait_drain(BAR(C::B_KVFULL + r % C::STAGES), (r / C::STAGES) & 1, p.timeout_ns);
      if (q_last >= 0) wait_drain(BAR(C::B_QFULL), q_last & 1, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ================================ MMA issuer ================================
    if (lane == 0) {
      uint32_t rc = 0, sj = 0;
      int n = 0;
      for (int ii = i_begin; ii < i_end; ++ii, ++n) {
        const WorkItem it = p.items[p.cta_items[ii]];
        if (!wait_bounded(BAR(C::B_QFULL), n & 1, guard, kWaitQFull)) break;
        tc_fence_after();
        const int T = C::NQ * it.job_count;
        uint32_t rk = 0, rv = 0;
        auto qk = [&](int t) -> bool {
          const int q = t % C::NQ;
          if (q == 0) {
            rk = rc;
            for (int h = 0; h < C::NCH; ++h, ++rc)
              if (!wait_bounded(BAR(C::B_KVFULL + rc % C::STAGES), (rc / C::STAGES) & 1, guard, kWaitKvFull))
                return false;
            tc_fence_after();
          }
          const uint32_t slot = (sj + t) & 1;
          const uint32_t qbase = sbase + C::OFF_Q + q * C::Q_BYTES;
#pragma unroll
          for (int kk = 0; kk < C::D / 16; ++kk) {
            const int col = kk * 16;
            const int h = col / C::CH, c = (col % C::CH) / 64, w = col % 64;
            const uint64_t a = sdesc(qbase + (col / 64) * C::BOX_BYTES + w * 2, 16, 1024);
            const uint64_t b = sdesc(sbase + C::OFF_RING + ((rk + h) % C::STAGES) * C::CHUNK_BYTES +
                                         c * C::BOX_BYTES + w * 2,
                                     16, 1024);
            mma_ss(tmem + 128 * slot, a, b, C::IDESC_QK, kk > 0 ? 1u : 0u);
          }
          mma_commit(BAR(C::B_SFULL + slot));
          if (q == C::NQ - 1)
            for (int h = 0; h < C::NCH; ++h) mma_commit(BAR(C::B_KVEMPTY + (rk + h) % C::STAGES));
          if (t == T - 1) mma_commit(BAR(C::B_QEMPTY));
          return true;
        };
        auto pv = [&](int u) -> bool {
          const int q = u % C::NQ;
          const uint32_t g = sj + u, slot = g & 1;
          if (!wait_bounded(BAR(C::B_PFULL + slot), (g >> 1) & 1, guard, kWaitPFull)) return false;
          if (u < C::NQ && !wait_bounded(BAR(C::B_OEMPTY + q), (n & 1) ^ 1, guard, kWaitOEmpty)) return false;
          if (q == 0) {
            rv = rc;
            for (int h = 0; h < C::NCH; ++h, ++rc)
              if (!wait_bounded(BAR(C::B_KVFULL + rc % C::STAGES), (rc / C::STAGES) & 1, guard, kWaitKvFull))
                return false;
          }
          tc_fence_after();
#pragma unroll
          for (int h = 0; h < C::NCH; ++h) {
            const uint32_t vbase = sbase + C::OFF_RING + ((rv + h) % C::STAGES) * C::CHUNK_BYTES;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t b = sdesc(vbase + kk * 2048, C::BOX_BYTES, 1024);
              mma_ts(tmem + C::TM_O + q * C::D + h * 128, tmem + 128 * slot + kk * 8, b, C::IDESC_PV,
                     (u < C::NQ && kk == 0) ? 0u : 1u);
            }
          }
          mma_commit(BAR(C::B_PVDONE + q));
          if (q == C::NQ - 1)
            for (int h = 0; h < C::NCH; ++h) mma_commit(BAR(C::B_KVEMPTY + (rv + h) % C::STAGES));
          return true;
        };
        bool ok = qk(0);
        if (ok && T > 1) ok = qk(1);
        for (int u = 0; ok && u < T; ++u) {
          ok = pv(u);
          if (ok && u + 2 < T) ok = qk(u + 2);
        }
        if (!ok) break;
        sj += T;
      }
      // all MMAs this thread issued complete before TMEM may be freed
      mma_commit(BAR(C::B_DRAIN));
      wait_drain(BAR(C::B_DRAIN), 0, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ================================ softmax warpgroup ================================
    const int q = warp / 4 - 1;                       // query tile of this warpgroup
    const int r = tid - 128 * (1 + q);                // row of the tile = TMEM lane
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const uint32_t t_o = tmem + lane_base + C::TM_O + q * C::D;
    const float sl2 = p.scale_log2;
    uint32_t sj = 0, pvc = 0;
    bool ok = true;
    for (int ii = i_begin; ok && ii < i_end; ++ii) {
      const WorkItem it = p.items[p.cta_items[ii]];
      const int T = C::NQ * it.job_count;
      float m_run = -INFINITY, l_run = 0.f;
      for (int t = q; t < T; t += C::NQ) {
        const uint32_t g = sj + t, slot = g & 1;
        const int mi = p.jobs[it.job_start + t / C::NQ].mask[q];
        uint4 bits = make_uint4(0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu);
        if (mi >= 0) bits = __ldg(p.mask_tiles + int64_t(mi) * 128 + r);
        else if (mi == kMaskNone) bits = make_uint4(0u, 0u, 0u, 0u);
        if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_SFULL + slot), (g >> 1) & 1, guard, kWaitSFull))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t t_s = tmem + lane_base + 128 * slot;
        float s[128];
        {
          uint32_t su[128];
          tmem_ld32x32(t_s + 0, su + 0);
          tmem_ld32x32(t_s + 32, su + 32);
          tmem_ld32x32(t_s + 64, su + 64);
          tmem_ld32x32(t_s + 96, su + 96);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(su[c]);
        }
        if (mi != kMaskFull) {
          const uint32_t wv[4] = {bits.x, bits.y, bits.z, bits.w};
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (!((wv[c >> 5] >> (c & 31)) & 1u)) s[c] = -INFINITY;
        }
        float mx = s[0];
#pragma unroll
        for (int c = 1; c < 128; ++c) mx = fmaxf(mx, s[c]);
        const float m_new = mx * sl2;
        const bool need = m_new > m_run + 8.0f;
        float alpha = 1.f;
        if (need) {
          alpha = ex2(m_run - m_new);
          m_run = m_new;
          l_run *= alpha;
        }
        const float mref = m_run == -INFINITY ? 0.f : m_run;
        float lsum = 0.f;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float p0 = ex2(fmaf(s[cc * 32 + 2 * e], sl2, -mref));
            const float p1 = ex2(fmaf(s[cc * 32 + 2 * e + 1], sl2, -mref));
            lsum += p0 + p1;
            pk[e] = pack_bf16(p0, p1);
          }
          tmem_st32x16(t_s + cc * 16, pk);
        }
        l_run += lsum;
        tmem_wait_st();
        if (t >= C::NQ) {
          // the previous P V of this tile must be done before O is touched or P is published
          if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_PVDONE + q), pvc & 1, guard, kWaitPvDone))) {
            ok = false;
            break;
          }
          ++pvc;
          tc_fence_after();
          if (__any_sync(0xffffffffu, need)) {
#pragma unroll 1
            for (int cc = 0; cc < C::D / 32; ++cc) {
              uint32_t o[32];
              tmem_ld32x32(t_o + cc * 32, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              tmem_st32x32(t_o + cc * 32, o);
            }
            tmem_wait_st();
          }
        }
        tc_fence_before();
        mbar_arrive(BAR(C::B_PFULL + slot));
      }
      if (!ok) break;
      // ---- epilogue: out = O / l, lse = ln(2) (m + log2 l) ----
      if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_PVDONE + q), pvc & 1, guard, kWaitPvDone))) break;
      ++pvc;
      tc_fence_after();
      const int lr = r % p.R, hh = r / p.R;
      const bool valid = lr < it.rows[q];
      const int64_t row = int64_t(it.tok[q] + lr) * p.hq + it.head[q] + hh;
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll 1
      for (int cc = 0; cc < C::D / 32; ++cc) {
        uint32_t o[32];
        tmem_ld32x32(t_o + cc * 32, o);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(p.out + row * C::D + cc * 32);
          dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          dst[2] = make_uint4(pk[8], pk[9], pk[10], pk[11]);
          dst[3] = make_uint4(pk[12], pk[13], pk[14], pk[15]);
        }
      }
      if (valid && p.lse) p.lse[row] = l_run > 0.f ? (m_run + log2f(l_run)) * 0.69314718055994531f : -INFINITY;
      tc_fence_before();
      mbar_arrive(BAR(C::B_OEMPTY + q));
      sj += T;
    }
  }
#undef BAR
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
}

// Rows of a problem without any key at all: out = 0, lse = -inf.
__global__ void fill_empty_kernel(float* lse, int64_t n) {
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x)
    lse[i] = -INFINITY;
}

// ---- host side ---------------------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

bool encode3d(CUtensorMap* tm, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t box2) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  const cuuint32_t box[3] = {64, 1, box2};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <class C>
attn_status_t launch(const attn_plan_t* plan, Params& p, cudaStream_t stream) {
  static std::once_flag once;
  static cudaError_t attr = cudaSuccess;
  std::call_once(once, [] {
    attr = cudaFuncSetAttribute(masked_attn_fwd_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                C::SMEM_BYTES);
  });
  if (attr != cudaSuccess) return ATTN_ERR_CUDA;
  masked_attn_fwd_kernel<C><<<plan->ctas, C::THREADS, C::SMEM_BYTES, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace
}  // namespace mfa

attn_status_t mfa_launch_forward(const attn_plan_t* plan, const void* q, const void* k, const void* v, void* out,
                                 float* lse, cudaStream_t stream) {
  using namespace mfa;
  const int D = plan->d;
  if (plan->total_kv_rows == 0) {
    // no key anywhere: every row is fully masked
    cudaError_t e = cudaMemsetAsync(out, 0, size_t(plan->total_q) * plan->hq * D * 2, stream);
    if (e == cudaSuccess && lse) {
      fill_empty_kernel<<<148, 256, 0, stream>>>(lse, plan->total_q * plan->hq);
      e = cudaGetLastError();
    }
    return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
  }
  Params p{};
  const uint32_t kv_box = plan->paged ? uint32_t(plan->page_size) : 128u;
  if (!encode3d(&p.tm_q, q, D, plan->hq, plan->total_q, uint32_t(plan->R)) ||
      !encode3d(&p.tm_k, k, D, plan->hkv, plan->total_kv_rows, kv_box) ||
      !encode3d(&p.tm_v, v, D, plan->hkv, plan->total_kv_rows, kv_box))
    return ATTN_ERR_CUDA;
  p.items = plan->d_items;
  p.jobs = plan->d_jobs;
  p.cta_off = plan->d_cta_off;
  p.cta_items = plan->d_cta_items;
  p.mask_tiles = plan->d_mask_tiles;
  p.page_table = plan->page_table;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.status = plan->d_status;
  p.hq = plan->hq;
  p.R = plan->R;
  p.hp = plan->hp;
  p.page_size = plan->page_size;
  p.num_pages = plan->num_pages;
  p.debug_flags = plan->debug_flags;
  p.scale_log2 = plan->scale * 1.4426950408889634f;
  p.timeout_ns = plan->timeout_ns;
  if (D == 64) {
    return plan->paged ? launch<Cfg<64, 2, 10, true>>(plan, p, stream) : launch<Cfg<64, 2, 10, false>>(plan, p, stream);
  } else if (D == 128) {
    return plan->paged ? launch<Cfg<128, 2, 5, true>>(plan, p, stream) : launch<Cfg<128, 2, 5, false>>(plan, p, stream);
  } else {
    return plan->paged ? launch<Cfg<256, 1, 5, true>>(plan, p, stream) : launch<Cfg<256, 1, 5, false>>(plan, p, stream);
  }
}

// ---- allocation-free forward ------------------------------------------------------------
// For embedders that may not allocate device memory: the plan of each call is copied into
// this fixed array instead of a cudaMalloc'd workspace. Host code never dereferences the
// symbol: it passes the address that cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[ATTN_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device, looked up once per device.
attn_status_t noalloc_scratch(int dev, void** out) {
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return ATTN_ERR_CUDA;
    g_noalloc_addr[dev] = ptr;
  }
  *out = g_noalloc_addr[dev];
  return ATTN_OK;
}
}  // namespace

extern "C" attn_status_t attn_masked_fwd_noalloc(const attn_problem_t* problem, const attn_mask_desc_t* mask,
                                                 const void* q, const void* k, const void* v, void* out,
                                                 float* lse, attn_stream_t stream_handle) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_handle);
  int dev = 0, num_sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return ATTN_ERR_CUDA;
  void* scratch = nullptr;
  attn_status_t st = noalloc_scratch(dev, &scratch);
  if (st != ATTN_OK) return st;
  mfa_host_plan hp;
  st = mfa_plan_host(problem, mask, num_sms, &hp);
  if (st != ATTN_OK) return st;
  if (hp.bytes.size() > size_t(ATTN_NOALLOC_SCRATCH_BYTES)) return ATTN_ERR_TOO_LARGE;
  if (hp.meta.total_q == 0) return ATTN_OK;
  if (!q || !k || !v || !out) return ATTN_ERR_INVALID_ARG;
  auto mis = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) != 0; };
  if (mis(q) || mis(k) || mis(v) || mis(out) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3)))
    return ATTN_ERR_INVALID_ARG;
  // the bytes start with a zeroed status word: each call clears what the previous one left
  if (cudaMemcpyAsync(scratch, hp.bytes.data(), hp.bytes.size(), cudaMemcpyHostToDevice, stream) != cudaSuccess)
    return ATTN_ERR_CUDA;
  char* base = static_cast<char*>(scratch);
  attn_plan_t& plan = hp.meta;
  plan.d_status = reinterpret_cast<int32_t*>(base);
  plan.d_items = reinterpret_cast<const mfa::WorkItem*>(base + hp.off_items);
  plan.d_jobs = reinterpret_cast<const mfa::Job*>(base + hp.off_jobs);
  plan.d_cta_off = reinterpret_cast<const int32_t*>(base + hp.off_cta_off);
  plan.d_cta_items = reinterpret_cast<const int32_t*>(base + hp.off_cta_items);
  plan.d_mask_tiles = reinterpret_cast<const uint4*>(base + hp.off_tiles);
  // (a copy from pageable host memory returns once the source has been staged, so the host
  // bytes may go away when this function returns)
  return mfa_launch_forward(&plan, q, k, v, out, lse, stream);
}
