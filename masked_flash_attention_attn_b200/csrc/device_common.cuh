// Device helpers shared by the forward (attn_fwd.cu) and backward (attn_bwd.cu) kernels:
// PTX wrappers for mbarriers with bounded waits, TMA, UMMA descriptors, tcgen05 MMA /
// commit / TMEM access, cluster addressing, packed fp32x2 arithmetic and bf16 packing.
// Included inside namespace mfa { namespace { ... } } of each translation unit.
#pragma once

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
  uint32_t abort_addr;       // this CTA's abort flag (shared::cta)
  uint32_t abort_peer;       // the cluster peer's abort flag (shared::cluster), 0 when alone
  int32_t* status;
  int64_t timeout_ns;
};

// Slow path of the bounded waits: spin until the phase completes, the abort flag is raised
// (returns false) or timeout_ns passes (raises this CTA's and the peer's flags, records `code`).
__device__ __forceinline__ bool wait_slow(uint32_t bar, uint32_t parity, const Guard& g, int32_t code) {
  const uint64_t t0 = gtime();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 16; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (ld_volatile_shared(g.abort_addr) != 0u) return false;
    if (gtime() - t0 > uint64_t(g.timeout_ns)) {
      st_volatile_shared(g.abort_addr, 1u);
      if (g.abort_peer) asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(g.abort_peer), "r"(1u) : "memory");
      atomicCAS(g.status, 0, code);
      return false;
    }
  }
}

// Wait for the phase of `parity` to complete; false when the CTA is aborting.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, const Guard& g, int32_t code) {
  if (mbar_try_wait(bar, parity)) return true;
  return wait_slow(bar, parity, g, code);
}

// Wait without looking at the abort flag (used to let in-flight async work land before
// the CTA exits); still bounded.
__device__ __forceinline__ void wait_drain(uint32_t bar, uint32_t parity, int64_t timeout_ns) {
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

// L2 eviction priority for the pair kernel's TMA loads: K/V tiles are re-read by every
// query tile of their (sequence, head), Q tiles once per item (measured: +0.7 % at d=256;
// the single-CTA kernel loads without hints, where they measured neutral to -3.5 %).
#ifndef MFA_L2_HINTS
#define MFA_L2_HINTS 1
#endif
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ void prefetch_l1(const void* ptr) {
  asm volatile("prefetch.global.L1 [%0];" ::"l"(ptr));
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* tm) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tm)) : "memory");
}

// Descriptors split into words: the high word (stride byte offset 1024, version 1, 128-byte
// swizzle) is the same for every operand here; the low word holds the start address and
// the leading byte offset, so stepping through a tile is one 32-bit add per operand.
constexpr uint32_t kDescHi = (1024u >> 4) | (1u << 14) | (2u << 29);
__device__ __forceinline__ uint32_t desc_lo(uint32_t addr, uint32_t lbo) {
  return ((addr & 0x3FFFFu) >> 4) | ((lbo >> 4) << 16);
}
__device__ __forceinline__ uint64_t desc_of(uint32_t lo) { return (uint64_t(kDescHi) << 32) | lo; }



__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// shared::cluster address of the same variable in cluster CTA `rank`
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Arrive on a barrier given by its shared::cluster address (this CTA's or the peer's).
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// Warp-level publication of TMEM writes to the pair leader: every lane has waited for its
// tcgen05.st and fenced them; after the warp converges one lane arrives (barrier count is
// one per warp of both CTAs).
__device__ __forceinline__ void warp_arrive_leader(uint32_t cluster_addr) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive_remote(cluster_addr);
}

// 2-SM MMAs of a CTA pair (mma2_*_x* in mma_groups.inc, issued by the pair's leader): A rows
// split over the two CTAs, B rows (N) split over the two CTAs, D rows split, all at the same
// offsets in both CTAs.


// arrive on the barrier at this offset in both CTAs of the pair when the MMAs complete
__device__ __forceinline__ void mma2_commit_both(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"(uint16_t(3))
      : "memory");
}

__device__ __forceinline__ void mma2_commit_self(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// TMA load into this CTA's shared memory whose completion is counted on the pair leader's
// barrier (`bar` is a shared::cluster address); no multicast.
__device__ __forceinline__ void tma2_load_3d(uint32_t dst, const CUtensorMap* tm, int32_t c0, int32_t c1, int32_t c2,
                                             uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void tma2_load_3d_hint(uint32_t dst, const CUtensorMap* tm, int32_t c0, int32_t c1,
                                                  int32_t c2, uint32_t bar, uint64_t pol) {
  if (!MFA_L2_HINTS) return tma2_load_3d(dst, tm, c0, c1, c2, bar);
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(c0), "r"(c1), "r"(c2), "r"(bar), "l"(pol)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

#include "tmem_ldst.inc"
#include "mma_groups.inc"

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the FMA/ALU pipes, for the share of the softmax exponentials that the kernel takes
// off the MUFU unit. Cody-Waite style reduction x = n + f, n = round(x) (the 1.5 * 2^23
// addition leaves n in the low mantissa bits), f in [-1/2, 1/2]; 2^f by the degree-3
// polynomial of least maximum relative error (Remez exchange; coefficients and the fit
// are produced by gen_exp2_poly.py next to this file, max relative error 7.5e-5); 2^n is
// applied by adding n to the exponent field. x is clamped at -125 so the result stays a
// normal float (>= ~2e-38, i.e. zero for every use here).
#define EXP2_POLY_C0 0x1.fff692p-1f  // 0.999928057
#define EXP2_POLY_C1 0x1.62f31ap-1f  // 0.693260968
#define EXP2_POLY_C2 0x1.f0de1ap-3f  // 0.242611125
#define EXP2_POLY_C3 0x1.c3f76p-5f   // 0.0551716685
__device__ __forceinline__ float exp2_poly(float x) {
  x = fmaxf(x, -125.0f);
  const float y = x + 12582912.0f;      // 1.5 * 2^23: y = 1.5 * 2^23 + round(x)
  const float f = x - (y - 12582912.0f);
  float p = fmaf(EXP2_POLY_C3, f, EXP2_POLY_C2);
  p = fmaf(p, f, EXP2_POLY_C1);
  p = fmaf(p, f, EXP2_POLY_C0);
  return __int_as_float(__float_as_int(p) + (__float_as_int(y) << 23));
}

// Packed fp32x2 arithmetic (sm_100): one instruction for two lanes of a float2.
__device__ __forceinline__ uint64_t pk2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void unpk2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// exp2_poly on a packed pair (same arithmetic as exp2_poly, two lanes per instruction).
__device__ __forceinline__ uint64_t exp2_poly2(float x0, float x1) {
  x0 = fmaxf(x0, -125.0f);
  x1 = fmaxf(x1, -125.0f);
  const uint64_t magic = pk2(12582912.0f, 12582912.0f);
  const uint64_t x = pk2(x0, x1);
  const uint64_t y = fadd2(x, magic);
  const uint64_t nmagic = pk2(-12582912.0f, -12582912.0f);
  const uint64_t r = fadd2(y, nmagic);             // round(x)
  float r0, r1;
  unpk2(r, r0, r1);
  const uint64_t f = fadd2(x, pk2(-r0, -r1));      // x - round(x)
  uint64_t p = ffma2(pk2(EXP2_POLY_C3, EXP2_POLY_C3), f, pk2(EXP2_POLY_C2, EXP2_POLY_C2));
  p = ffma2(p, f, pk2(EXP2_POLY_C1, EXP2_POLY_C1));
  p = ffma2(p, f, pk2(EXP2_POLY_C0, EXP2_POLY_C0));
  float p0, p1, y0, y1;
  unpk2(p, p0, p1);
  unpk2(y, y0, y1);
  return pk2(__int_as_float(__float_as_int(p0) + (__float_as_int(y0) << 23)),
             __int_as_float(__float_as_int(p1) + (__float_as_int(y1) << 23)));
}

// Three-operand maximum (sm_100 adds the 3-input form of max.f32).
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Four fp32 -> four e4m3 in one word (round to nearest even, saturating at +-448); `a0` in
// the lowest byte (the lowest key index). cvt's first source lands in the upper byte.
__device__ __forceinline__ uint32_t pack_e4m3x4(float a0, float a1, float a2, float a3) {
  uint16_t lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(a1), "f"(a0));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(a3), "f"(a2));
  return uint32_t(lo) | (uint32_t(hi) << 16);
}

// Two fp32 -> one bf16x2 word (round to nearest even); `lo` lands in the low half, which
// is the lower column / key index in every layout used here.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// ---- host: tensor maps ---------------------------------------------------------------------
// 3-D bf16 tensor map over [d2][d1][d0] (d0 contiguous), boxes of {64, 1, box2} elements with
// the 128-byte swizzle: one 64-column slice of box2 rows of one head.
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

// 3-D byte (e4m3) tensor map: dims d0 (contiguous) x d1 x d2, row strides s1 / s2 bytes
// (multiples of 16), boxes {b0, b1, b2} with the 128-byte swizzle (b0 = 128).
bool encode3d_u8(CUtensorMap* tm, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1, uint64_t s2,
                 uint32_t b0, uint32_t b1, uint32_t b2) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {s1, s2};
  const cuuint32_t box[3] = {b0, b1, b2};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
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

// Runs `set` (a kernel's launch attributes) once per device and returns its result on every
// later call from that device: the attributes belong to one device's context, and a process
// may drive several GPUs. Each call site's lambda type gives it its own flags.
template <class F>
cudaError_t once_per_device(F set) {
  constexpr int kDevices = 64;
  static std::once_flag flags[kDevices];
  static cudaError_t result[kDevices];
  int dev = 0;
  const cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kDevices) return cudaErrorInvalidDevice;
  std::call_once(flags[dev], [&] { result[dev] = set(); });
  return result[dev];
}
