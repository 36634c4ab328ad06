// Masked attention forward for sm_100a (B200).
//
// One persistent CTA (or CTA pair) per SM walks its list of work items (built by the
// planner). A work item is two 128-row query tiles that share one key/value head and one
// run of key tiles; empty key tiles never appear in the run, full key tiles carry no mask,
// partial ones carry the index of a 2 KiB tile-transposed bit mask. Three kernels:
//
//   masked_attn_fwd_kernel       (head_dim 64 / 128 in bf16, 128 in e4m3): the two query
//       tiles take turns in one S accumulator in TMEM, P has a TMEM slot of its own per tile,
//       Q K^T and P V are issued by two different threads (see the kernel's comment).
//   masked_attn_fwd_pair_kernel  (head_dim 256, bf16 or e4m3): a CTA pair, one query tile per
//       CTA, 2-SM MMAs (cta_group::2) so each SM streams half of every K and V tile; S double
//       buffered per tile, P written over S.
//
// Every wait on an mbarrier is bounded (globaltimer). When a wait expires the thread
// records ATTN_ERR_TIMEOUT in the plan's status word, raises a shared abort flag that
// ends every other wait, lets its own copies / MMAs in flight complete, and the CTA
// frees its TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "attn_internal.h"
#include "attn_testing.h"

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
  float* part_o;       // split-KV partial slots (kSlotRows x D fp32 each), or null
  float* part_lse;     // split-KV partial lse (kSlotRows fp32 per slot), or null
  int32_t* status;
  int32_t hq, R, hp, page_size, num_pages, debug_flags;
  float scale_log2;
  float v_scale;       // e4m3 forward: the value tensor's scale (1 for bf16)
  int64_t timeout_ns;
};

#include "device_common.cuh"

// ---- per-row softmax steps shared by both kernels ---------------------------------------
// One thread owns one row (= one TMEM lane). m_run is the reference maximum in the
// scaled log2 domain (scores * scale * log2 e); it is raised only when a tile's maximum
// exceeds it by more than 8, so P <= 2^8 and O / l are rescaled rarely (exact either way:
// O and l always share the same reference).
struct RowState {
  float m_run, l_run;
};

// S row (128 fp32 columns at t_s) -> masked online-softmax step -> P (bf16, written over
// the first 64 columns of t_s). Returns the factor alpha by which O and l must be
// multiplied (1 when the reference did not move); `need` tells whether it moved.
// FP8: P is written as e4m3, four per TMEM column (columns 0 .. 31), instead of bf16 pairs.
template <int EMU, bool FP8 = false>
__device__ __forceinline__ float softmax_tile(uint32_t t_s, int mi, const uint4& bits, float sl2, RowState& st,
                                              bool& need) {
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
  // row maximum: eight independent chains of 3-input max, then a small tree (one thread
  // owns the row, so a single 127-long dependent chain would cost its full latency)
  float m8[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) m8[k] = fmaxf(s[k], s[k + 8]);
#pragma unroll
  for (int j = 1; j < 8; ++j)
#pragma unroll
    for (int k = 0; k < 8; ++k) m8[k] = max3f(m8[k], s[16 * j + k], s[16 * j + 8 + k]);
  const float mx = max3f(max3f(m8[0], m8[1], m8[2]), max3f(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
  const float m_new = mx * sl2;
  need = m_new > st.m_run + 8.0f;
  float alpha = 1.f;
  if (need) {
    alpha = ex2(st.m_run - m_new);
    st.m_run = m_new;
    st.l_run *= alpha;
  }
  const float mref = st.m_run == -INFINITY ? 0.f : st.m_run;
  const uint64_t sl2x2 = pk2(sl2, sl2), nm2 = pk2(-mref, -mref);
  uint64_t lsum2[4] = {pk2(0.f, 0.f), pk2(0.f, 0.f), pk2(0.f, 0.f), pk2(0.f, 0.f)};  // 4 independent sums
  uint32_t p8[FP8 ? 32 : 1];
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) {
    uint32_t pk[16];
    float pf[FP8 ? 32 : 1];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      float x0, x1;
      unpk2(ffma2(pk2(s[cc * 32 + 2 * e], s[cc * 32 + 2 * e + 1]), sl2x2, nm2), x0, x1);
      uint64_t p01;
      if ((e & 7) < EMU) {
        p01 = exp2_poly2(x0, x1);
      } else {
        p01 = pk2(ex2(x0), ex2(x1));
      }
      lsum2[e & 3] = fadd2(lsum2[e & 3], p01);
      float p0, p1;
      unpk2(p01, p0, p1);
      if constexpr (FP8) {
        pf[2 * e] = p0;
        pf[2 * e + 1] = p1;
      } else {
        pk[e] = pack_bf16(p0, p1);
      }
    }
    if constexpr (FP8) {
#pragma unroll
      for (int w = 0; w < 8; ++w) p8[cc * 8 + w] = pack_e4m3x4(pf[4 * w], pf[4 * w + 1], pf[4 * w + 2], pf[4 * w + 3]);
    } else {
      tmem_st32x16(t_s + cc * 16, pk);
    }
  }
  if constexpr (FP8) tmem_st32x32(t_s, p8);
  {
    float a, b;
    unpk2(fadd2(fadd2(lsum2[0], lsum2[1]), fadd2(lsum2[2], lsum2[3])), a, b);
    st.l_run += a + b;
  }
  tmem_wait_st();
  return alpha;
}

// O row (D fp32 columns at t_o) *= alpha; warp-collective.
template <int D>
__device__ __forceinline__ void rescale_o(uint32_t t_o, float alpha) {
#pragma unroll 1
  for (int cc = 0; cc < D / 32; ++cc) {
    uint32_t o[32];
    tmem_ld32x32(t_o + cc * 32, o);
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
    tmem_st32x32(t_o + cc * 32, o);
  }
  tmem_wait_st();
}

// out = O / l (bf16), lse = ln 2 * (m + log2 l); rows that saw no key get 0 and -inf.
// A row saw a key iff its reference maximum is finite (the polynomial exp2 leaves ~2^-125,
// not 0, for masked entries, so l > 0 alone does not tell). Warp-collective TMEM reads;
// the global stores are guarded by `valid`.
template <int D>
__device__ __forceinline__ void store_row(uint32_t t_o, const RowState& st, bool valid, int64_t row,
                                          __nv_bfloat16* out, float* lse, float oscale = 1.f) {
  const bool seen = st.m_run != -INFINITY;
  const float inv = seen ? oscale / st.l_run : 0.f;
#pragma unroll 1
  for (int cc = 0; cc < D / 32; ++cc) {
    uint32_t o[32];
    tmem_ld32x32(t_o + cc * 32, o);
    tmem_wait_ld();
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e)
      pk[e] = pack_bf16(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
    if (valid) {
      uint4* dst = reinterpret_cast<uint4*>(out + row * D + cc * 32);
      dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
      dst[2] = make_uint4(pk[8], pk[9], pk[10], pk[11]);
      dst[3] = make_uint4(pk[12], pk[13], pk[14], pk[15]);
    }
  }
  if (valid && lse) lse[row] = seen ? (st.m_run + log2f(st.l_run)) * 0.69314718055994531f : -INFINITY;
}

// Split-KV: the row's result over this item's key range, out / l in fp32 and its lse
// (natural log), into partial slot row `srow`; merged later by merge_partials_kernel.
template <int D>
__device__ __forceinline__ void store_partial(uint32_t t_o, const RowState& st, bool valid, int64_t srow, float* po,
                                              float* plse, float oscale = 1.f) {
  const bool seen = st.m_run != -INFINITY;
  const float inv = seen ? oscale / st.l_run : 0.f;
#pragma unroll 1
  for (int cc = 0; cc < D / 32; ++cc) {
    uint32_t o[32];
    tmem_ld32x32(t_o + cc * 32, o);
    tmem_wait_ld();
    if (valid) {
      float4* dst = reinterpret_cast<float4*>(po + srow * D + cc * 32);
#pragma unroll
      for (int e = 0; e < 8; ++e)
        dst[e] = make_float4(__uint_as_float(o[4 * e]) * inv, __uint_as_float(o[4 * e + 1]) * inv,
                             __uint_as_float(o[4 * e + 2]) * inv, __uint_as_float(o[4 * e + 3]) * inv);
    }
  }
  if (valid) plse[srow] = seen ? (st.m_run + log2f(st.l_run)) * 0.69314718055994531f : -INFINITY;
}

// Paged K/V: the slots of a sequence's last page past its last key hold whatever the cache
// holds there, possibly NaN or Inf. Their scores are masked (P = 0), but 0 x NaN is NaN in
// P V, so before the P V of a key tile that reaches past the keys, the V rows of those
// slots are zeroed in shared memory: rows [r0, r1) of a V chunk (nbox 128-byte boxes of
// 128 rows, 16 KiB apart; the 128-byte swizzle permutes 16-byte pieces inside a row, so a
// whole row is the same 128 bytes). `lanes` threads starting at `lane` share the stores;
// `remote` (a cluster peer's shared::cluster address of the chunk) is zeroed as well when
// not 0. The stores are made visible to the tensor core's async proxy before returning.
__device__ __forceinline__ void zero_v_rows(uint32_t chunk, uint32_t remote, int nbox, int r0, int r1, int lane,
                                            int lanes) {
  const int n = (r1 - r0) * nbox * 8;   // 16-byte pieces
  for (int i = lane; i < n; i += lanes) {
    const int row = r0 + i / (nbox * 8), rem = i % (nbox * 8);
    const uint32_t off = uint32_t((rem >> 3) * 16384 + row * 128 + (rem & 7) * 16);
    asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(chunk + off), "r"(0u) : "memory");
    if (remote) asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(remote + off), "r"(0u) : "memory");
  }
  asm volatile("fence.proxy.async;" ::: "memory");
}

// Rows [r0, r1) of key tile kt to zero: the tail of the sequence's last page, when the tile
// reaches past the last key (rows from the page count on come from out-of-bounds boxes and
// are zeros already). r0 >= r1 when there is nothing to zero.
__device__ __forceinline__ void v_tail_rows(int kt, int kv_len, int npages, int page_size, int& r0, int& r1) {
  r0 = kv_len - kt * 128;
  r1 = npages * page_size - kt * 128;
  r1 = r1 < 128 ? r1 : 128;
  if (r0 < 0) r0 = r1;
}

// ---- the kernel ----------------------------------------------------------------------------

enum : int32_t {
  kWaitQEmpty = 0x100, kWaitKvEmpty, kWaitQFull, kWaitKvFull, kWaitPFull, kWaitOEmpty, kWaitSFull, kWaitPvDone
};

// ================================ shared-S kernel (head_dim 64 / 128 bf16, 128 e4m3) ================================
// One persistent CTA per SM, two 128-row query tiles per work item. The two query tiles take
// turns in ONE S accumulator (TMEM columns 0-127): a softmax warpgroup frees it as soon as it
// has read its scores into registers, so the next Q K^T (of the other tile) runs while it
// computes; P goes to a slot of its own per tile (columns 128 + 64 t, bf16 pairs), O of tile t
// sits at 256 + t D. Q K^T and P V are issued by two different threads, so a wait of one
// never idles the tensor core while the other has work:
//   warp 0       TMA producer: Q tiles once per item, then K(0), [K(1), V(0)], [K(2), V(1)],
//                ..., V(J-1) through a ring of STAGES chunks (a chunk = a 128-key K or V tile).
//   warp 1       Q K^T issuer: for key tile j, S = Q0 K(j)^T, then (once softmax 0 has read
//                S) S = Q1 K(j)^T; releases K(j).
//   warp 2       P V issuer: O_t += P_t V(j) for t = 0, 1 once P_t is published; releases V(j).
//   warp 3       idle (holds its warpgroup's TMEM lane quarter).
//   warpgroup 1+t  softmax of query tile t: one thread per row reads S, frees it, applies the
//                row's mask bits (partial tiles), updates the online max / sum, writes P into
//                its slot once the previous P V of the tile is done, rescales O when the
//                running maximum grows by more than 2^8, and finally writes out / lse.
// FP8_: e4m3 Q and K (one 128-byte box per 128-row tile), V transposed per head
// ([Hkv][d][keys]: a chunk is d = 128 rows x 128 keys), .kind::f8f6f4 MMAs of K = 32, and P
// quantised to e4m3 (four per TMEM column: a 32-column P slot); head_dim 128, contiguous K/V.
template <int D_, bool PAGED_, int EMU_ = 0, bool FP8_ = false>
struct SCfg {
  static constexpr int D = D_, EMU = EMU_;
  static constexpr bool PAGED = PAGED_;
  static constexpr bool FP8 = FP8_;
  static constexpr int NBOX = FP8 ? 1 : D / 64;       // 128-byte boxes per Q tile and per K / V chunk
  static constexpr int BOX_BYTES = 128 * 128;         // 128 rows x 128 bytes
  static constexpr int Q_BYTES = NBOX * BOX_BYTES;
  static constexpr int CHUNK_BYTES = NBOX * BOX_BYTES;
  static constexpr int STAGES = FP8 ? 12 : D == 128 ? 5 : 10;
  static constexpr int P_COLS = FP8 ? 32 : 64;        // TMEM columns of a P slot
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_RING = 2 * Q_BYTES;
  static constexpr int OFF_BAR = OFF_RING + STAGES * CHUNK_BYTES;
  static constexpr int B_QFULL = 0, B_QEMPTY = 1, B_KVFULL = 2, B_KVEMPTY = B_KVFULL + STAGES,
                       B_SFULL = B_KVEMPTY + STAGES, B_SFREE = B_SFULL + 2, B_PFULL = B_SFREE + 2,
                       B_PVDONE = B_PFULL + 2, B_OEMPTY = B_PVDONE + 2, B_DRAIN = B_OEMPTY + 2, NBAR = B_DRAIN + 2;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;  // [0] TMEM base, [1] abort flag
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int THREADS = 384;
  static constexpr int REG_LOW = 64, REG_HIGH = 208;
  static constexpr int REG_SPLIT_TOTAL = 128 * REG_LOW + 256 * REG_HIGH;
  static constexpr int TM_S = 0, TM_P = 128, TM_O = 256;
  static constexpr uint32_t AB_TYPES = FP8 ? 0u : (1u << 7) | (1u << 10);   // bf16 (1) or e4m3 (0)
  static constexpr uint32_t IDESC_QK =  // M=128, N=128, both K-major, fp32 accumulate
      (1u << 4) | AB_TYPES | (uint32_t(128 >> 3) << 17) | (uint32_t(128 >> 4) << 24);
  static constexpr uint32_t IDESC_PV =  // M=128, N=D, A (P) from TMEM, B: V MN-major (bf16), V^T K-major (e4m3)
      (1u << 4) | AB_TYPES | (FP8 ? 0u : (1u << 16)) | (uint32_t(D >> 3) << 17) | (uint32_t(128 >> 4) << 24);
  static_assert(D == 64 || D == 128, "shared-S kernel: head_dim 64 or 128");
  static_assert(!FP8 || (D == 128 && !PAGED), "e4m3 shared-S kernel: head_dim 128, contiguous K/V");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(TM_O + 2 * D <= 512, "TMEM budget");
};

// Position of K(j) / V(j) of an item with J key tiles in the producer's order
// K(0), [K(1), V(0)], [K(2), V(1)], ..., [K(J-1), V(J-2)], V(J-1) (2 J chunks).
__device__ __forceinline__ int k_pos(int j) { return j == 0 ? 0 : 2 * j - 1; }
__device__ __forceinline__ int v_pos(int j, int J) { return j == J - 1 ? 2 * J - 1 : 2 * j + 2; }

// Softmax step of a shared-S tile: the row's 128 scores at t_s (fp32) into registers, then
// `freed()` (the S accumulator may be overwritten), mask / max / exponentials / row sum, and
// P (bf16 pairs) into pk[64]. Returns the factor by which O and l must be multiplied.
// FP8: P as e4m3, four per word (pk[0 .. 31]) instead of bf16 pairs (pk[0 .. 63]).
template <int EMU, bool FP8, class Freed>
__device__ __forceinline__ float softmax_regs(uint32_t t_s, int mi, const uint4& bits, float sl2, RowState& st,
                                              bool& need, uint32_t (&pk)[64], Freed freed) {
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
  freed();
  if (mi != kMaskFull) {
    const uint32_t wv[4] = {bits.x, bits.y, bits.z, bits.w};
#pragma unroll
    for (int c = 0; c < 128; ++c)
      if (!((wv[c >> 5] >> (c & 31)) & 1u)) s[c] = -INFINITY;
  }
  float m8[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) m8[k] = fmaxf(s[k], s[k + 8]);
#pragma unroll
  for (int j = 1; j < 8; ++j)
#pragma unroll
    for (int k = 0; k < 8; ++k) m8[k] = max3f(m8[k], s[16 * j + k], s[16 * j + 8 + k]);
  const float mx = max3f(max3f(m8[0], m8[1], m8[2]), max3f(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
  const float m_new = mx * sl2;
  need = m_new > st.m_run + 8.0f;
  float alpha = 1.f;
  if (need) {
    alpha = ex2(st.m_run - m_new);
    st.m_run = m_new;
    st.l_run *= alpha;
  }
  const float mref = st.m_run == -INFINITY ? 0.f : st.m_run;
  const uint64_t sl2x2 = pk2(sl2, sl2), nm2 = pk2(-mref, -mref);
  uint64_t lsum2[4] = {pk2(0.f, 0.f), pk2(0.f, 0.f), pk2(0.f, 0.f), pk2(0.f, 0.f)};
  float pprev0 = 0.f, pprev1 = 0.f;
#pragma unroll
  for (int e = 0; e < 64; ++e) {
    float x0, x1;
    unpk2(ffma2(pk2(s[2 * e], s[2 * e + 1]), sl2x2, nm2), x0, x1);
    uint64_t p01;
    if ((e & 7) < EMU) p01 = exp2_poly2(x0, x1);
    else p01 = pk2(ex2(x0), ex2(x1));
    lsum2[e & 3] = fadd2(lsum2[e & 3], p01);
    float p0, p1;
    unpk2(p01, p0, p1);
    if constexpr (FP8) {
      if (e & 1) pk[e >> 1] = pack_e4m3x4(pprev0, pprev1, p0, p1);
      pprev0 = p0;
      pprev1 = p1;
    } else {
      pk[e] = pack_bf16(p0, p1);
    }
  }
  float a, b;
  unpk2(fadd2(fadd2(lsum2[0], lsum2[1]), fadd2(lsum2[2], lsum2[3])), a, b);
  st.l_run += a + b;
  return alpha;
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1) masked_attn_fwd_kernel(const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem_raw + (sbase - raw) + C::OFF_MISC);
  const uint32_t bar0 = sbase + C::OFF_BAR;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Guard guard{smem_u32(misc + 1), 0u, p.status, p.timeout_ns};
#define BAR(i) (bar0 + 8u * uint32_t(i))

  if (tid == 0) {
    mbar_init(BAR(C::B_QFULL), 1);
    mbar_init(BAR(C::B_QEMPTY), 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(BAR(C::B_KVFULL + s), 1);
      mbar_init(BAR(C::B_KVEMPTY + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(BAR(C::B_SFULL + t), 1);
      mbar_init(BAR(C::B_SFREE + t), 4);      // one arrival per softmax warp
      mbar_init(BAR(C::B_PFULL + t), 4);
      mbar_init(BAR(C::B_PVDONE + t), 1);
      mbar_init(BAR(C::B_OEMPTY + t), 4);
      mbar_init(BAR(C::B_DRAIN + t), 1);
    }
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

  if (warp < 4) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REG_LOW));
  if (warp == 0) {
    // ================================ TMA producer ================================
    // The whole warp runs the loop: lane 0 issues the Q copies and the contiguous K / V
    // boxes; with a paged cache lane i issues the boxes of the chunk's page i (a single thread
    // issuing many small boxes is limited by its own issue rate; one lane per page measured
    // faster than one lane per box). Waits are taken by every lane and agreed with a vote.
    {
      uint32_t rc = 0;
      int n = 0, q_last = -1;
      for (int ii = i_begin; ii < i_end; ++ii, ++n) {
        const WorkItem it = p.items[p.cta_items[ii]];
        if constexpr (C::PAGED) {
          if (lane == 0) {
            prefetch_l1(p.page_table + it.k_base);
            if (ii + 1 < i_end) prefetch_l1(p.page_table + p.items[p.cta_items[ii + 1]].k_base);
          }
        }
        if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_QEMPTY), (n & 1) ^ 1, guard, kWaitQEmpty))) break;
        if (!((p.debug_flags & 1) && n == 0)) {
          q_last = n;
          if (lane == 0) {
            mbar_expect_tx(BAR(C::B_QFULL), 2 * C::Q_BYTES);
            for (int t = 0; t < 2; ++t)
              for (int hh = 0; hh < p.hp; ++hh)
                for (int c = 0; c < C::NBOX; ++c)
                  tma_load_3d(sbase + C::OFF_Q + t * C::Q_BYTES + c * C::BOX_BYTES + hh * p.R * 128, &p.tm_q,
                              c * (C::FP8 ? 128 : 64), it.head[t] + hh, it.tok[t], BAR(C::B_QFULL));
          }
        }
        auto load_tile = [&](bool is_v, int j) -> bool {
          const int kt = p.jobs[it.job_start + j].k_tile;
          const CUtensorMap* tm = is_v ? &p.tm_v : &p.tm_k;
          const uint32_t slot = rc % C::STAGES;
          if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_KVEMPTY + slot), ((rc / C::STAGES) & 1) ^ 1, guard,
                                                    kWaitKvEmpty)))
            return false;
          const uint32_t dst = sbase + C::OFF_RING + slot * C::CHUNK_BYTES;
          if (lane == 0) mbar_expect_tx(BAR(C::B_KVFULL + slot), C::CHUNK_BYTES);
          if constexpr (C::FP8) {
            // K: 128 keys x 128 bytes; V^T ([Hkv][d][keys]): d = 128 rows x 128 keys
            if (lane == 0) {
              if (is_v) tma_load_3d(dst, tm, it.vt_base + kt * 128, 0, it.kv_head, BAR(C::B_KVFULL + slot));
              else tma_load_3d(dst, tm, 0, it.kv_head, it.k_base + kt * 128, BAR(C::B_KVFULL + slot));
            }
          } else if constexpr (!C::PAGED) {
            if (lane == 0)
              for (int c = 0; c < C::NBOX; ++c)
                tma_load_3d(dst + c * C::BOX_BYTES, tm, c * 64, it.kv_head, it.k_base + kt * 128,
                            BAR(C::B_KVFULL + slot));
          } else {
            const int ps = p.page_size, ppt = 128 / ps;
            if (lane == 0 && !is_v) {
              const int ahead = (kt + 2) * ppt;
              if (ahead < it.npages) prefetch_l1(p.page_table + it.k_base + ahead);
            }
            __syncwarp();   // the expected byte count is posted before any of the chunk's copies
            if (lane < ppt) {   // lane = page of the chunk
              const int idx = kt * ppt + lane;
              const int32_t page = idx < it.npages ? __ldg(p.page_table + it.k_base + idx) : -1;
              int32_t row = p.num_pages * ps;  // fully out of bounds: the box reads zeros
              if (page >= 0 && page < p.num_pages) row = page * ps;
              for (int c = 0; c < C::NBOX; ++c)
                tma_load_3d(dst + c * C::BOX_BYTES + lane * ps * 128, tm, c * 64, it.kv_head, row,
                            BAR(C::B_KVFULL + slot));
            }
          }
          ++rc;
          return true;
        };
        const int J = it.job_count;
        bool ok = load_tile(false, 0);
        for (int j = 1; ok && j < J; ++j) {
          ok = load_tile(false, j);
          if (ok) ok = load_tile(true, j - 1);
        }
        if (ok) ok = load_tile(true, J - 1);
        if (!ok) break;
      }
      if (lane == 0) {
        for (uint32_t r = rc > uint32_t(C::STAGES) ? rc - C::STAGES : 0u; r < rc; ++r)
          wait_drain(BAR(C::B_KVFULL + r % C::STAGES), (r / C::STAGES) & 1, p.timeout_ns);
        if (q_last >= 0) wait_drain(BAR(C::B_QFULL), q_last & 1, p.timeout_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ================================ Q K^T issuer ================================
    if (lane == 0) {
      uint32_t base = 0;              // ring position of the item's first chunk
      uint32_t nfree[2] = {0u, 0u};   // S-free phases consumed per tile
      uint32_t produced = 0;          // Q K^T groups issued so far
      int n = 0;
      for (int ii = i_begin; ii < i_end; ++ii, ++n) {
        const int J = p.items[p.cta_items[ii]].job_count;
        if (!wait_bounded(BAR(C::B_QFULL), n & 1, guard, kWaitQFull)) break;
        bool ok = true;
        for (int j = 0; ok && j < J; ++j) {
          const uint32_t rk = base + uint32_t(k_pos(j));
          if (!wait_bounded(BAR(C::B_KVFULL + rk % C::STAGES), (rk / C::STAGES) & 1, guard, kWaitKvFull)) {
            ok = false;
            break;
          }
          const uint32_t klo = desc_lo(sbase + C::OFF_RING + (rk % C::STAGES) * C::CHUNK_BYTES, 16);
          for (int t = 0; t < 2; ++t) {
            // the previous scores in S (the other tile's) have been read
            if (produced > 0) {
              const int prev = t ^ 1;
              if (!wait_bounded(BAR(C::B_SFREE + prev), nfree[prev] & 1, guard, kWaitSFull)) {
                ok = false;
                break;
              }
              ++nfree[prev];
            }
            tc_fence_after();
            const uint32_t qlo = desc_lo(sbase + C::OFF_Q + t * C::Q_BYTES, 16);
            if constexpr (C::FP8) mma8_ss_x4_k128(tmem + C::TM_S, desc_of(qlo), desc_of(klo), C::IDESC_QK, 0u);
            else if constexpr (C::D == 128) mma_ss_x8_k128(tmem + C::TM_S, desc_of(qlo), desc_of(klo), C::IDESC_QK, 0u);
            else mma_ss_x4_k64(tmem + C::TM_S, desc_of(qlo), desc_of(klo), C::IDESC_QK, 0u);
            mma_commit(BAR(C::B_SFULL + t));
            ++produced;
          }
          if (!ok) break;
          mma_commit(BAR(C::B_KVEMPTY + rk % C::STAGES));
        }
        if (!ok) break;
        mma_commit(BAR(C::B_QEMPTY));
        base += 2u * uint32_t(J);
      }
      mma_commit(BAR(C::B_DRAIN + 0));
      wait_drain(BAR(C::B_DRAIN + 0), 0, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ================================ P V issuer ================================
    if (lane == 0) {
      uint32_t base = 0;
      uint32_t pc[2] = {0u, 0u};      // P phases consumed per tile
      int n = 0;
      for (int ii = i_begin; ii < i_end; ++ii, ++n) {
        const WorkItem* itp = p.items + p.cta_items[ii];
        const int J = itp->job_count, job_start = itp->job_start;
        const int kv_len = C::PAGED ? itp->kv_len : 0, npages = C::PAGED ? itp->npages : 0;
        bool ok = true;
        for (int j = 0; ok && j < J; ++j) {
          const uint32_t rv = base + uint32_t(v_pos(j, J));
          if (!wait_bounded(BAR(C::B_KVFULL + rv % C::STAGES), (rv / C::STAGES) & 1, guard, kWaitKvFull)) {
            ok = false;
            break;
          }
          const uint32_t vbase = sbase + C::OFF_RING + (rv % C::STAGES) * C::CHUNK_BYTES;
          if constexpr (C::PAGED) {
            int r0, r1;
            v_tail_rows(p.jobs[job_start + j].k_tile, kv_len, npages, p.page_size, r0, r1);
            if (r0 < r1) zero_v_rows(vbase, 0u, C::NBOX, r0, r1, 0, 1);
          }
          for (int t = 0; t < 2; ++t) {
            if (!wait_bounded(BAR(C::B_PFULL + t), pc[t] & 1, guard, kWaitPFull)) {
              ok = false;
              break;
            }
            ++pc[t];
            if (j == 0 && !wait_bounded(BAR(C::B_OEMPTY + t), (n & 1) ^ 1, guard, kWaitOEmpty)) {
              ok = false;
              break;
            }
            tc_fence_after();
            if constexpr (C::FP8)
              mma8_ts_x4_k128(tmem + C::TM_O + t * C::D, tmem + C::TM_P + C::P_COLS * t, desc_of(desc_lo(vbase, 16)),
                              C::IDESC_PV, j == 0 ? 0u : 1u);
            else
              mma_ts_x8(tmem + C::TM_O + t * C::D, tmem + C::TM_P + C::P_COLS * t,
                        desc_of(desc_lo(vbase, C::BOX_BYTES)), C::IDESC_PV, j == 0 ? 0u : 1u);
            mma_commit(BAR(C::B_PVDONE + t));
          }
          if (!ok) break;
          mma_commit(BAR(C::B_KVEMPTY + rv % C::STAGES));
        }
        if (!ok) break;
        base += 2u * uint32_t(J);
      }
      mma_commit(BAR(C::B_DRAIN + 1));
      wait_drain(BAR(C::B_DRAIN + 1), 0, p.timeout_ns);
    }
    __syncwarp();
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::REG_HIGH));
    // ================================ softmax warpgroup of query tile q ================================
    const int q = warp / 4 - 1;
    const int r = tid - 128 * (1 + q);                // row of the tile = TMEM lane
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const uint32_t t_o = tmem + lane_base + C::TM_O + q * C::D;
    const uint32_t t_p = tmem + lane_base + C::TM_P + C::P_COLS * q;
    const float sl2 = p.scale_log2;
    uint32_t sc = 0, pc = 0;   // S phases consumed, P published
    bool ok = true;
    auto wait_pv = [&]() -> bool {   // the P V of the last P published is done
      if (pc == 0) return true;
      return __all_sync(0xffffffffu, wait_bounded(BAR(C::B_PVDONE + q), (pc - 1) & 1, guard, kWaitPvDone));
    };
    for (int ii = i_begin; ok && ii < i_end; ++ii) {
      const WorkItem it = p.items[p.cta_items[ii]];
      const int J = it.job_count;
      RowState st{-INFINITY, 0.f};
      for (int j = 0; j < J; ++j) {
        const int mi = p.jobs[it.job_start + j].mask[q];
        uint4 bits = make_uint4(0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu);
        if (mi >= 0) bits = __ldg(p.mask_tiles + int64_t(mi) * 128 + r);
        else if (mi == kMaskNone) bits = make_uint4(0u, 0u, 0u, 0u);
        if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_SFULL + q), sc & 1, guard, kWaitSFull))) {
          ok = false;
          break;
        }
        ++sc;
        tc_fence_after();
        bool need;
        uint32_t pk[64];
        const float alpha = softmax_regs<C::EMU, C::FP8>(tmem + lane_base + C::TM_S, mi, bits, sl2, st, need, pk, [&] {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(BAR(C::B_SFREE + q));
        });
        // the previous P V of this tile has read its P and added into O
        if (!wait_pv()) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (j > 0 && __any_sync(0xffffffffu, need)) rescale_o<C::D>(t_o, alpha);
        if constexpr (C::FP8) {
          tmem_st32x32(t_p, pk);
        } else {
          tmem_st32x16(t_p + 0, pk + 0);
          tmem_st32x16(t_p + 16, pk + 16);
          tmem_st32x16(t_p + 32, pk + 32);
          tmem_st32x16(t_p + 48, pk + 48);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(C::B_PFULL + q));
        ++pc;
      }
      if (!ok) break;
      // ---- epilogue ----
      if (!wait_pv()) break;
      tc_fence_after();
      const int lr = r % p.R, hh = r / p.R;
      if (it.part < 0)
        store_row<C::D>(t_o, st, lr < it.rows[q], int64_t(it.tok[q] + lr) * p.hq + it.head[q] + hh, p.out, p.lse,
                        p.v_scale);
      else
        store_partial<C::D>(t_o, st, lr < it.rows[q], int64_t(it.part + q) * kSlotRows + r, p.part_o, p.part_lse,
                            p.v_scale);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::B_OEMPTY + q));
    }
  }
#undef BAR
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
}

// ================================ cluster-pair kernel (head_dim 256) ================================
// Two CTAs on the two SMs of a pair cooperate on one work item: CTA r owns query tile r
// (128 rows) and its TMEM rows; the pair's leader (r = 0) issues 2-SM MMAs of M = 256:
//   S  = Q K^T : A = each CTA's Q tile, B = each CTA's HALF of the key tile (keys 64r..64r+63)
//   O += P V   : A = each CTA's P (TMEM), B = each CTA's HALF of the value columns
// so every CTA streams half of K and half of V per key tile, and one query tile per CTA
// keeps two S buffers (the next S = Q K^T runs while the softmax works on the current one).
// Both CTAs' TMA loads count on the leader's "full" barriers; the leader's commits arrive
// on both CTAs' barriers; the softmax warpgroups of both CTAs arrive on the leader's "P
// ready" and "O free" barriers. No TMA load multicasts.
// FP8_: e4m3 Q, K and V^T ([Hkv][d][keys]; each CTA reads the d / 2 rows of its V half),
// .kind::f8f6f4 2-SM MMAs, P in e4m3.
template <int D_, int STAGES_, bool PAGED_, int EMU_ = 0, bool FP8_ = false>
struct PairCfg {
  static constexpr int D = D_, STAGES = STAGES_, EMU = EMU_;
  static constexpr bool PAGED = PAGED_;
  static constexpr bool FP8 = FP8_;
  static constexpr int BOX_COLS = FP8 ? 128 : 64;  // elements per 128-byte box row
  static constexpr int QBOX = D / BOX_COLS;        // 128-byte boxes of a Q tile and of a K half
  // boxes of a V half: bf16 d / 2 columns in 64-column boxes (MN-major); e4m3 one box of d / 2
  // V^T rows x 128 keys (K-major)
  static constexpr int VBOX = FP8 ? 1 : D / 128;
  static constexpr int Q_BYTES = QBOX * 128 * 128;
  static constexpr int KH_BOX = 64 * 128;          // 64 keys x 128 bytes
  static constexpr int VH_BOX = 128 * 128;         // 128 keys x 128 bytes
  static constexpr int SLOT_BYTES = QBOX * KH_BOX; // == VBOX * VH_BOX
  static_assert(QBOX * KH_BOX == VBOX * VH_BOX, "K and V halves fill one ring slot");
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_RING = Q_BYTES;
  static constexpr int OFF_BAR = OFF_RING + STAGES * SLOT_BYTES;
  static constexpr int B_QFULL = 0, B_QEMPTY = 1, B_KVFULL = 2, B_KVEMPTY = B_KVFULL + STAGES,
                       B_SFULL = B_KVEMPTY + STAGES, B_PFULL = B_SFULL + 2, B_PVDONE = B_PFULL + 2,
                       B_OEMPTY = B_PVDONE + 1, B_DRAIN = B_OEMPTY + 1, NBAR = B_DRAIN + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int THREADS = 256;
  static constexpr int TM_O = 256;
  static constexpr uint32_t AB_TYPES = FP8 ? 0u : (1u << 7) | (1u << 10);   // bf16 (1) or e4m3 (0)
  static constexpr uint32_t IDESC_QK =  // M=256 (pair), N=128, fp32 accumulate, both K-major
      (1u << 4) | AB_TYPES | (uint32_t(128 >> 3) << 17) | (uint32_t(256 >> 4) << 24);
  static constexpr uint32_t IDESC_PV =  // M=256, N=D, A (P) from TMEM; B: V MN-major (bf16), V^T K-major (e4m3)
      (1u << 4) | AB_TYPES | (FP8 ? 0u : (1u << 16)) | (uint32_t(D >> 3) << 17) | (uint32_t(256 >> 4) << 24);
  static_assert(!FP8 || (D == 256 && !PAGED), "e4m3 pair kernel: head_dim 256, contiguous K/V");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(256 + D <= 512, "TMEM budget");
};

template <class C>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(C::THREADS, 1)
    masked_attn_fwd_pair_kernel(const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem_raw + (sbase - raw) + C::OFF_MISC);
  const uint32_t bar0 = sbase + C::OFF_BAR;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
#define BAR(i) (bar0 + 8u * uint32_t(i))
  const uint32_t lbar0 = mapa_shared(bar0, 0);   // the leader's barriers, cluster addresses
#define LBAR(i) (lbar0 + 8u * uint32_t(i))
  const Guard guard{smem_u32(misc + 1), mapa_shared(smem_u32(misc + 1), rank ^ 1u), p.status, p.timeout_ns};

  if (tid == 0) {
    mbar_init(BAR(C::B_QFULL), 1);
    mbar_init(BAR(C::B_QEMPTY), 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(BAR(C::B_KVFULL + s), 1);
      mbar_init(BAR(C::B_KVEMPTY + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(BAR(C::B_SFULL + s), 1);
      mbar_init(BAR(C::B_PFULL + s), 8);   // one arrival per softmax warp of both CTAs
    }
    mbar_init(BAR(C::B_PVDONE), 1);
    mbar_init(BAR(C::B_OEMPTY), 8);
    mbar_init(BAR(C::B_DRAIN), 1);
    misc[1] = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tmap(&p.tm_q);
    prefetch_tmap(&p.tm_k);
    prefetch_tmap(&p.tm_v);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(misc))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  const int cl = blockIdx.x / 2;
  const int i_begin = p.cta_off[cl], i_end = p.cta_off[cl + 1];

  if (warp == 0) {
    // ================================ TMA producer (both CTAs) ================================
    // The whole warp runs the loop (waits agreed with a vote); lane 0 issues the Q copies
    // and the contiguous K / V boxes, and with a paged cache every box of a half-chunk (page,
    // 64-column block) has its own lane: one thread's TMA issue rate bounds many small boxes.
    {
      const uint64_t pol_kv = l2_policy_evict_last(), pol_q = l2_policy_evict_first();
      uint32_t rc = 0;
      int n = 0, q_last = -1;
      for (int ii = i_begin; ii < i_end; ++ii, ++n) {
        const WorkItem it = p.items[p.cta_items[ii]];
        if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_QEMPTY), (n & 1) ^ 1, guard, kWaitQEmpty))) break;
        if (!((p.debug_flags & 1) && n == 0)) {
          q_last = n;
          if (lane == 0) {
            if (leader) mbar_expect_tx(BAR(C::B_QFULL), 2 * C::Q_BYTES);
            for (int hh = 0; hh < p.hp; ++hh)
              for (int c = 0; c < C::QBOX; ++c)
                tma2_load_3d_hint(sbase + C::OFF_Q + c * 16384 + hh * p.R * 128, &p.tm_q, c * C::BOX_COLS,
                                  it.head[rank] + hh, it.tok[rank], LBAR(C::B_QFULL), pol_q);
          }
        }
        const int T = it.job_count;
        auto load_half = [&](bool is_v, int j) -> bool {
          const int kt = p.jobs[it.job_start + j].k_tile;
          const uint32_t slot = rc % C::STAGES;
          if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_KVEMPTY + slot), ((rc / C::STAGES) & 1) ^ 1, guard,
                                                    kWaitKvEmpty)))
            return false;
          if (leader && lane == 0) mbar_expect_tx(BAR(C::B_KVFULL + slot), 2 * C::SLOT_BYTES);
          const uint32_t dst = sbase + C::OFF_RING + slot * C::SLOT_BYTES;
          const uint32_t fb = LBAR(C::B_KVFULL + slot);
          // K half: keys kt*128 + 64 rank .. +63, all D columns; V half: all 128 keys,
          // columns rank*D/2 .. +D/2
          const int key0 = kt * 128 + (is_v ? 0 : 64 * int(rank));
          const int nkeys = is_v ? 128 : 64;
          const int nbox = is_v ? C::VBOX : C::QBOX;
          const int box_bytes = is_v ? C::VH_BOX : C::KH_BOX;
          const int col0 = is_v ? int(rank) * (C::D / 2) : 0;
          const CUtensorMap* tm = is_v ? &p.tm_v : &p.tm_k;
          if constexpr (C::FP8) {
            // K half: 64 keys x two 128-byte boxes; V^T half: d / 2 rows x 128 keys
            if (lane != 0) {
            } else if (is_v)
              tma2_load_3d_hint(dst, tm, it.vt_base + kt * 128, int(rank) * (C::D / 2), it.kv_head, fb, pol_kv);
            else
              for (int c = 0; c < nbox; ++c)
                tma2_load_3d_hint(dst + c * box_bytes, tm, c * C::BOX_COLS, it.kv_head, it.k_base + key0, fb, pol_kv);
          } else if constexpr (!C::PAGED) {
            if (lane == 0)
              for (int c = 0; c < nbox; ++c)
                tma2_load_3d_hint(dst + c * box_bytes, tm, col0 + c * C::BOX_COLS, it.kv_head, it.k_base + key0, fb,
                                  pol_kv);
          } else {
            const int ps = p.page_size;
            const int rows = ps < nkeys ? ps : nkeys;  // rows per box
            const int nb = nkeys / rows;               // boxes per 64-column block
            if (!is_v && lane == 0) {
              const int ahead = ((kt + 2) * 128) / ps;   // page-table line of the key tile two ahead
              if (ahead < it.npages) prefetch_l1(p.page_table + it.k_base + ahead);
            }
            __syncwarp();   // this CTA's expected byte count is posted before its copies
            if (lane < nb * nbox) {   // lane = (page block of the half-chunk, 64-column box)
              const int pg = lane / nbox, c = lane % nbox, idx = (key0 + pg * rows) / ps;
              const int32_t page = idx < it.npages ? __ldg(p.page_table + it.k_base + idx) : -1;
              int32_t row = p.num_pages * ps;  // fully out of bounds: the box reads zeros
              if (page >= 0 && page < p.num_pages) row = page * ps + (key0 + pg * rows) % ps;
              tma2_load_3d_hint(dst + c * box_bytes + pg * rows * 128, tm, col0 + c * C::BOX_COLS, it.kv_head, row, fb,
                                pol_kv);
            }
          }
          ++rc;
          return true;
        };
        bool ok = load_half(false, 0);
        if (ok && T > 1) ok = load_half(false, 1);
        for (int u = 0; ok && u < T; ++u) {
          ok = load_half(true, u);
          if (ok && u + 2 < T) ok = load_half(false, u + 2);
        }
        if (!ok) break;
      }
      // let the copies land before the CTA may exit: the leader's barriers count both CTAs' bytes
      if (leader && lane == 0) {
        for (uint32_t r = rc > uint32_t(C::STAGES) ? rc - C::STAGES : 0u; r < rc; ++r)
          wait_drain(BAR(C::B_KVFULL + r % C::STAGES), (r / C::STAGES) & 1, p.timeout_ns);
        if (q_last >= 0) wait_drain(BAR(C::B_QFULL), q_last & 1, p.timeout_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ================================ MMA issuer (leader only) ================================
    if (lane == 0 && leader) {
      uint32_t rc = 0, sj = 0;
      int n = 0;
      for (int ii = i_begin; ii < i_end; ++ii, ++n) {
        const WorkItem it = p.items[p.cta_items[ii]];
        if (!wait_bounded(BAR(C::B_QFULL), n & 1, guard, kWaitQFull)) break;
        tc_fence_after();
        const int T = it.job_count;
        auto qk = [&](int t) -> bool {
          const uint32_t slot = (sj + t) & 1, rk = rc;
          if (!wait_bounded(BAR(C::B_KVFULL + rc % C::STAGES), (rc / C::STAGES) & 1, guard, kWaitKvFull))
            return false;
          ++rc;
          tc_fence_after();
          const uint32_t qlo = desc_lo(sbase + C::OFF_Q, 16);
          const uint32_t klo = desc_lo(sbase + C::OFF_RING + (rk % C::STAGES) * C::SLOT_BYTES, 16);
          const uint32_t d_s = tmem + 128 * slot;
          static_assert(C::D == 256, "pair kernel issue groups are laid out for head_dim 256");
          if constexpr (C::FP8) mma2_8_ss_x8_k256(d_s, desc_of(qlo), desc_of(klo), C::IDESC_QK, 0u);
          else mma2_ss_x16_k256(d_s, desc_of(qlo), desc_of(klo), C::IDESC_QK, 0u);
          mma2_commit_both(BAR(C::B_KVEMPTY + rk % C::STAGES));
          mma2_commit_both(BAR(C::B_SFULL + slot));
          if (t == T - 1) mma2_commit_both(BAR(C::B_QEMPTY));
          return true;
        };
        auto pv = [&](int u) -> bool {
          const uint32_t g = sj + u, slot = g & 1, rv = rc;
          if (!wait_bounded(BAR(C::B_PFULL + slot), (g >> 1) & 1, guard, kWaitPFull)) return false;
          if (u == 0 && !wait_bounded(BAR(C::B_OEMPTY), (n & 1) ^ 1, guard, kWaitOEmpty)) return false;
          if (!wait_bounded(BAR(C::B_KVFULL + rc % C::STAGES), (rc / C::STAGES) & 1, guard, kWaitKvFull))
            return false;
          ++rc;
          tc_fence_after();
          const uint32_t vbase = sbase + C::OFF_RING + (rv % C::STAGES) * C::SLOT_BYTES;
          if constexpr (C::PAGED) {
            // both CTAs' V halves: the leader writes the peer's through its cluster address
            int r0, r1;
            v_tail_rows(p.jobs[it.job_start + u].k_tile, it.kv_len, it.npages, p.page_size, r0, r1);
            if (r0 < r1) zero_v_rows(vbase, mapa_shared(vbase, 1), C::VBOX, r0, r1, 0, 1);
          }
          const uint32_t a_p = tmem + 128 * slot, acc0 = u == 0 ? 0u : 1u;
          if constexpr (C::FP8) mma2_8_ts_x4(tmem + C::TM_O, a_p, desc_of(desc_lo(vbase, 16)), C::IDESC_PV, acc0);
          else mma2_ts_x8(tmem + C::TM_O, a_p, desc_of(desc_lo(vbase, C::VH_BOX)), C::IDESC_PV, acc0);
          mma2_commit_both(BAR(C::B_KVEMPTY + rv % C::STAGES));
          mma2_commit_both(BAR(C::B_PVDONE));
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
      mma2_commit_self(BAR(C::B_DRAIN));
      wait_drain(BAR(C::B_DRAIN), 0, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ================================ softmax warpgroup (both CTAs) ================================
    const int r = tid - 128;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const uint32_t t_o = tmem + lane_base + C::TM_O;
    const float sl2 = p.scale_log2;
    uint32_t sj = 0, pvc = 0;
    bool ok = true;
    for (int ii = i_begin; ok && ii < i_end; ++ii) {
      const WorkItem it = p.items[p.cta_items[ii]];
      const int T = it.job_count;
      RowState st{-INFINITY, 0.f};
      for (int t = 0; t < T; ++t) {
        const uint32_t g = sj + t, slot = g & 1;
        const int mi = p.jobs[it.job_start + t].mask[rank];
        uint4 bits = make_uint4(0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu);
        if (mi >= 0) bits = __ldg(p.mask_tiles + int64_t(mi) * 128 + r);
        else if (mi == kMaskNone) bits = make_uint4(0u, 0u, 0u, 0u);
        if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_SFULL + slot), (g >> 1) & 1, guard, kWaitSFull))) {
          ok = false;
          break;
        }
        tc_fence_after();
        bool need;
        const float alpha = softmax_tile<C::EMU, C::FP8>(tmem + lane_base + 128 * slot, mi, bits, sl2, st, need);
        if (t >= 1) {
          if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_PVDONE), pvc & 1, guard, kWaitPvDone))) {
            ok = false;
            break;
          }
          ++pvc;
          tc_fence_after();
          if (__any_sync(0xffffffffu, need)) rescale_o<C::D>(t_o, alpha);
        }
        tc_fence_before();
        warp_arrive_leader(LBAR(C::B_PFULL + slot));
      }
      if (!ok) break;
      if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_PVDONE), pvc & 1, guard, kWaitPvDone))) break;
      ++pvc;
      tc_fence_after();
      const int lr = r % p.R, hh = r / p.R;
      if (it.part < 0)
        store_row<C::D>(t_o, st, lr < it.rows[rank], int64_t(it.tok[rank] + lr) * p.hq + it.head[rank] + hh, p.out,
                        p.lse, p.v_scale);
      else
        store_partial<C::D>(t_o, st, lr < it.rows[rank], int64_t(it.part + int(rank)) * kSlotRows + r, p.part_o,
                            p.part_lse, p.v_scale);
      tc_fence_before();
      warp_arrive_leader(LBAR(C::B_OEMPTY));
      sj += T;
    }
  }
#undef LBAR
#undef BAR
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
}

__global__ void exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t n) {
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x)
    y[i] = exp2_poly(x[i]);
}

// Split-KV merge. With lse_r the partial lse of key range r and o_r its out / l:
// lse = m + ln sum_r exp(lse_r - m) (m = max_r lse_r), out = sum_r exp(lse_r - lse) o_r;
// a row that saw no key in any range gets out = 0, lse = -inf. Grid (merge tiles,
// kSlotRows / 8): one warp per row; the lanes first share out the range weights (kept in
// shared memory), then each lane sums the ranges for its 4-column groups.
constexpr int kMergeRowsPerBlock = 8;
__global__ void __launch_bounds__(32 * kMergeRowsPerBlock) merge_partials_kernel(
    const MergeTile* __restrict__ tiles, const float* __restrict__ part_o, const float* __restrict__ part_lse, int D,
    int R, int hq, __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
  __shared__ float wsh[kMergeRowsPerBlock][kMaxSplits];
  const MergeTile t = tiles[blockIdx.x];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.y * kMergeRowsPerBlock + warp;
  const int lr = r % R, hh = r / R;
  if (lr >= t.rows) return;
  const int64_t orow = int64_t(t.tok + lr) * hq + t.head + hh;
  float m = -INFINITY;
  for (int k = lane; k < t.nsplit; k += 32) m = fmaxf(m, part_lse[int64_t(t.slot0 + k * t.stride) * kSlotRows + r]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (m == -INFINITY) {
    for (int c = 4 * lane; c < D; c += 128) *reinterpret_cast<uint2*>(out + orow * D + c) = make_uint2(0u, 0u);
    if (lse && lane == 0) lse[orow] = -INFINITY;
    return;
  }
  float wsum = 0.f;
  for (int k = lane; k < t.nsplit; k += 32) {
    const float w = expf(part_lse[int64_t(t.slot0 + k * t.stride) * kSlotRows + r] - m);
    wsh[warp][k] = w;
    wsum += w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
  __syncwarp();
  const float inv = 1.f / wsum;
  for (int c = 4 * lane; c < D; c += 128) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int k = 0; k < t.nsplit; ++k) {
      const float w = wsh[warp][k];
      const float4 o = *reinterpret_cast<const float4*>(part_o + (int64_t(t.slot0 + k * t.stride) * kSlotRows + r) * D + c);
      acc.x = fmaf(w, o.x, acc.x);
      acc.y = fmaf(w, o.y, acc.y);
      acc.z = fmaf(w, o.z, acc.z);
      acc.w = fmaf(w, o.w, acc.w);
    }
    *reinterpret_cast<uint2*>(out + orow * D + c) =
        make_uint2(pack_bf16(acc.x * inv, acc.y * inv), pack_bf16(acc.z * inv, acc.w * inv));
  }
  if (lse && lane == 0) lse[orow] = m + logf(wsum);
}

// Rows of a problem without any key at all: out = 0, lse = -inf.
__global__ void fill_empty_kernel(float* lse, int64_t n) {
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x)
    lse[i] = -INFINITY;
}

// ---- host side ---------------------------------------------------------------------------

// Column pairs (of every 8) whose exponentials the d <= 128 kernels take off the MUFU unit.
#ifndef MFA_EMU_D128
#define MFA_EMU_D128 0
#endif


template <class C>
attn_status_t launch_sharedS(const attn_plan_t* plan, Params& p, cudaStream_t stream) {
  const cudaError_t attr = once_per_device([] {
    cudaError_t e = cudaFuncSetAttribute(masked_attn_fwd_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::SMEM_BYTES);
    if (e == cudaSuccess) {
      // setmaxnreg.inc draws on the registers the block was launched with: the split must fit
      cudaFuncAttributes fa{};
      e = cudaFuncGetAttributes(&fa, masked_attn_fwd_kernel<C>);
      if (e == cudaSuccess && fa.numRegs * C::THREADS < C::REG_SPLIT_TOTAL) e = cudaErrorInvalidConfiguration;
    }
    return e;
  });
  if (attr != cudaSuccess) return ATTN_ERR_CUDA;
  masked_attn_fwd_kernel<C><<<plan->ctas, C::THREADS, C::SMEM_BYTES, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <class C>
attn_status_t launch_pair(const attn_plan_t* plan, Params& p, cudaStream_t stream) {
  const cudaError_t attr = once_per_device([] {
    return cudaFuncSetAttribute(masked_attn_fwd_pair_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                C::SMEM_BYTES);
  });
  if (attr != cudaSuccess) return ATTN_ERR_CUDA;
  // grid = 2 CTAs per work unit; the kernel's cluster shape (2, 1, 1) is compiled in
  masked_attn_fwd_pair_kernel<C><<<2 * plan->ctas, C::THREADS, C::SMEM_BYTES, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace
}  // namespace mfa

namespace {

// out = 0 and lse = -inf everywhere: a problem without any key.
attn_status_t forward_no_keys(const attn_plan_t* plan, void* out, float* lse, cudaStream_t stream) {
  cudaError_t e = cudaMemsetAsync(out, 0, size_t(plan->total_q) * plan->hq * plan->d * 2, stream);
  if (e == cudaSuccess && lse) {
    mfa::fill_empty_kernel<<<148, 256, 0, stream>>>(lse, plan->total_q * plan->hq);
    e = cudaGetLastError();
  }
  return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// The plan's work list, masks and partial slots, the outputs and the scalars into Params.
void plan_params(const attn_plan_t* plan, void* out, float* lse, mfa::Params& p) {
  p.items = plan->d_items;
  p.jobs = plan->d_jobs;
  p.cta_off = plan->d_cta_off;
  p.cta_items = plan->d_cta_items;
  p.mask_tiles = plan->d_mask_tiles;
  p.page_table = plan->page_table;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.part_o = plan->d_part_o;
  p.part_lse = plan->d_part_lse;
  p.status = plan->d_status;
  p.hq = plan->hq;
  p.R = plan->R;
  p.hp = plan->hp;
  p.page_size = plan->page_size;
  p.num_pages = plan->num_pages;
  p.debug_flags = plan->debug_flags;
  p.scale_log2 = plan->scale * 1.4426950408889634f;
  p.v_scale = 1.f;
  p.timeout_ns = plan->timeout_ns;
}

// Split-KV: merge the partial results of the split query tiles (after the forward kernel).
attn_status_t merge_if_split(const attn_plan_t* plan, void* out, float* lse, cudaStream_t stream) {
  using namespace mfa;
  if (plan->n_merge == 0) return ATTN_OK;
  const dim3 grid(plan->n_merge, kSlotRows / kMergeRowsPerBlock);
  merge_partials_kernel<<<grid, 32 * kMergeRowsPerBlock, 0, stream>>>(plan->d_merge, plan->d_part_o, plan->d_part_lse,
                                                                     plan->d, plan->R, plan->hq,
                                                                     static_cast<__nv_bfloat16*>(out), lse);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

attn_status_t mfa_launch_forward(const attn_plan_t* plan, const void* q, const void* k, const void* v, void* out,
                                 float* lse, cudaStream_t stream) {
  using namespace mfa;
  const int D = plan->d;
  if (plan->total_kv_rows == 0) return forward_no_keys(plan, out, lse, stream);
  Params p{};
  // rows per K / V box: a page, a whole 128-key tile, or (pair kernel) a 64-key half tile
  const uint32_t ps = uint32_t(plan->page_size);
  uint32_t k_box = plan->paged ? ps : 128u, v_box = k_box;
  if (plan->cluster == 2) k_box = k_box < 64u ? k_box : 64u;
  if (!encode3d(&p.tm_q, q, D, plan->hq, plan->total_q, uint32_t(plan->R)) ||
      !encode3d(&p.tm_k, k, D, plan->hkv, plan->total_kv_rows, k_box) ||
      !encode3d(&p.tm_v, v, D, plan->hkv, plan->total_kv_rows, v_box))
    return ATTN_ERR_CUDA;
  plan_params(plan, out, lse, p);
  attn_status_t st;
  if (D == 64) {
    st = plan->paged ? launch_sharedS<SCfg<64, true, MFA_EMU_D128>>(plan, p, stream)
                     : launch_sharedS<SCfg<64, false, MFA_EMU_D128>>(plan, p, stream);
  } else if (D == 128) {
    st = plan->paged ? launch_sharedS<SCfg<128, true, MFA_EMU_D128>>(plan, p, stream)
                     : launch_sharedS<SCfg<128, false, MFA_EMU_D128>>(plan, p, stream);
  } else {
    st = plan->paged ? launch_pair<PairCfg<256, 5, true>>(plan, p, stream)
                     : launch_pair<PairCfg<256, 5, false>>(plan, p, stream);
  }
  return st != ATTN_OK ? st : merge_if_split(plan, out, lse, stream);
}

// e4m3 forward (head_dim 128, contiguous K/V, single-CTA kernel): q, k bytes
// [rows][heads][128]; vt bytes [Hkv][128][ldv] (V transposed per head); the scores are
// scale * q_scale * k_scale * (q8 . k8), the output v_scale * (P8 . vt8) / l.
attn_status_t mfa_launch_forward_fp8(const attn_plan_t* plan, const void* q, const void* k, const void* vt,
                                     int64_t ldv, float q_scale, float k_scale, float v_scale, void* out, float* lse,
                                     cudaStream_t stream) {
  using namespace mfa;
  const bool pair = plan->d == 256;
  if ((plan->d != 128 && !pair) || plan->paged || plan->cluster != (pair ? 2 : 1)) return ATTN_ERR_UNSUPPORTED;
  if (plan->total_kv_rows == 0) return forward_no_keys(plan, out, lse, stream);
  Params p{};
  const uint64_t D = uint64_t(plan->d);
  // K boxes: a 128-key tile (single-CTA kernel) or a 64-key half (pair); V^T boxes: d or d / 2 rows
  const uint32_t k_rows = pair ? 64u : 128u, vt_rows = uint32_t(pair ? D / 2 : D);
  if (!encode3d_u8(&p.tm_q, q, D, plan->hq, plan->total_q, D, D * plan->hq, 128, 1, uint32_t(plan->R)) ||
      !encode3d_u8(&p.tm_k, k, D, plan->hkv, plan->total_kv_rows, D, D * plan->hkv, 128, 1, k_rows) ||
      !encode3d_u8(&p.tm_v, vt, uint64_t(plan->vt_keys), D, plan->hkv, uint64_t(ldv), uint64_t(ldv) * D, 128, vt_rows,
                   1))
    return ATTN_ERR_CUDA;
  plan_params(plan, out, lse, p);
  p.scale_log2 = plan->scale * q_scale * k_scale * 1.4426950408889634f;
  p.v_scale = v_scale;
  // With e4m3 MMAs the exponentials weigh twice as much as in bf16: two column pairs of every
  // eight take the FMA-pipe polynomial (+4.5 % at d = 256, +3 % on the chunk-causal d = 128
  // workload, neutral on the block-dense one).
  const attn_status_t st = pair ? launch_pair<PairCfg<256, 10, false, 2, true>>(plan, p, stream)
                                : launch_sharedS<SCfg<128, false, 2, true>>(plan, p, stream);
  return st != ATTN_OK ? st : merge_if_split(plan, out, lse, stream);
}

namespace mfa {
namespace {
// V [rows][Hkv][d] (bytes) -> V^T [Hkv][d][ldv] with sequence b's keys at columns
// vt_off[b] .. (128-aligned starts) and zeros in the gaps; 32 x 32 byte tiles through
// shared memory, one 32-column tile of one head per block.
__global__ void transpose_v_kernel(const uint8_t* __restrict__ v, uint8_t* __restrict__ vt,
                                   const int32_t* __restrict__ cu_k, const int32_t* __restrict__ vt_off, int batch,
                                   int hkv, int d, int64_t ldv) {
  __shared__ uint8_t tile[32][33];
  const int c0 = blockIdx.x * 32;   // transposed column (padded key index)
  const int d0 = blockIdx.y * 32, h = blockIdx.z;
  const int tx = threadIdx.x, ty = threadIdx.y;
  for (int i = ty; i < 32; i += 8) {
    const int c = c0 + i;
    int lo = 0, hi = batch;   // the sequence b with vt_off[b] <= c < vt_off[b + 1]
    while (hi - lo > 1) {
      const int mid = (lo + hi) / 2;
      if (vt_off[mid] <= c) lo = mid;
      else hi = mid;
    }
    const int local = c - vt_off[lo];
    const int64_t row = int64_t(cu_k[lo]) + local;
    tile[i][tx] = (c < vt_off[batch] && row < cu_k[lo + 1]) ? v[(row * hkv + h) * d + d0 + tx] : uint8_t(0);
  }
  __syncthreads();
  for (int i = ty; i < 32; i += 8) {
    const int c = c0 + tx;
    if (c < vt_off[batch]) vt[(int64_t(h) * d + d0 + i) * ldv + c] = tile[tx][i];
  }
}
}  // namespace
}  // namespace mfa

attn_status_t mfa_transpose_v(const attn_plan_t* plan, const void* v, void* vt, int64_t ldv, cudaStream_t stream) {
  if (plan->vt_keys == 0 || plan->batch == 0) return ATTN_OK;
  const dim3 grid(uint32_t((plan->vt_keys + 31) / 32), uint32_t(plan->d / 32), uint32_t(plan->hkv)), block(32, 8);
  mfa::transpose_v_kernel<<<grid, block, 0, stream>>>(static_cast<const uint8_t*>(v), static_cast<uint8_t*>(vt),
                                                      plan->d_cu_k, plan->d_vt_off, plan->batch, plan->hkv, plan->d,
                                                      ldv);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

extern "C" attn_status_t attn_test_exp2_poly(const float* x, float* y, int64_t n, attn_stream_t stream) {
  if (n < 0 || (n > 0 && (!x || !y))) return ATTN_ERR_INVALID_ARG;
  if (n == 0) return ATTN_OK;
  mfa::exp2_poly_kernel<<<296, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, y, n);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
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
// test hook (attn_test_noalloc_debug): debug flags and wait limit of the following calls
std::atomic<int32_t> g_noalloc_debug_flags{0};
std::atomic<int64_t> g_noalloc_timeout_ns{2000000000LL};

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
  // No plan survives this call, so an in-kernel wait that expires cannot be reported through a
  // status query. Instead lse starts as NaN: every row the kernel completes overwrites it with
  // a finite value or -inf, so rows still NaN afterwards are the ones that were not computed.
  if (lse && cudaMemsetAsync(lse, 0xFF, size_t(hp.meta.total_q) * size_t(hp.meta.hq) * sizeof(float), stream) !=
                 cudaSuccess)
    return ATTN_ERR_CUDA;
  char* base = static_cast<char*>(scratch);
  attn_plan_t& plan = hp.meta;
  plan.d_status = reinterpret_cast<int32_t*>(base);
  plan.d_items = reinterpret_cast<const mfa::WorkItem*>(base + hp.off_items);
  plan.d_jobs = reinterpret_cast<const mfa::Job*>(base + hp.off_jobs);
  plan.d_cta_off = reinterpret_cast<const int32_t*>(base + hp.off_cta_off);
  plan.d_cta_items = reinterpret_cast<const int32_t*>(base + hp.off_cta_items);
  plan.d_mask_tiles = reinterpret_cast<const uint4*>(base + hp.off_tiles);
  plan.debug_flags = g_noalloc_debug_flags.load();
  plan.timeout_ns = g_noalloc_timeout_ns.load();
  // (a copy from pageable host memory returns once the source has been staged, so the host
  // bytes may go away when this function returns)
  return mfa_launch_forward(&plan, q, k, v, out, lse, stream);
}

extern "C" attn_status_t attn_test_noalloc_debug(int32_t flags, int64_t timeout_ns) {
  if (flags < 0 || timeout_ns <= 0) return ATTN_ERR_INVALID_ARG;
  g_noalloc_debug_flags.store(flags);
  g_noalloc_timeout_ns.store(timeout_ns);
  return ATTN_OK;
}
