// Internal definitions shared by the libbsa.so translation units: the
// derived geometry of a problem, the layout-buffer map, and thin wrappers
// over the sm_100a PTX used by the kernels (mbarrier, TMA, tcgen05).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/bsa.h"

namespace bsa {

constexpr int kBlock = 64;       // tokens per block
// blocks per sequence the attention kernel's on-chip step table can hold
// (16-bit entries: a 13-bit key block and 3 flags)
constexpr int kAttnMaxBlocks = 6144;

// Everything a kernel needs to know about a problem (plain integers).
struct Geo {
  int B, h, d;
  int T, H, W, Tv, Hv, Wv;
  int nseg;
  int seg_len[BSA_MAX_PREFIX_SEGMENTS];
  int seg_off[BSA_MAX_PREFIX_SEGMENTS];
  int P, N, Nv;
  int nbp, nbv, nb;
  int keep, kcap;
  int mode;
  int nreg;   // dynamic regions per batch element (0 in fixed mode)
  float tau, scale;
  int stall_pv;  // test hook: the attention kernel issues no PV (see bsa_debug_stall_pv)
};

// Byte offsets of the sections of the layout buffer (each 256-B aligned).
struct LayoutMap {
  size_t perm, iperm, bmask, bcount, codes, bfull, total;
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

__host__ __device__ inline LayoutMap layout_map(const Geo& g) {
  LayoutMap m;
  size_t off = 0;
  m.perm = off;   off = align256(off + sizeof(int32_t) * size_t(g.B) * g.N);
  m.iperm = off;  off = align256(off + sizeof(int32_t) * size_t(g.B) * g.N);
  m.bmask = off;  off = align256(off + sizeof(uint64_t) * size_t(g.B) * g.nb);
  m.bcount = off; off = align256(off + sizeof(int32_t) * size_t(g.B) * g.nb);
  m.codes = off;  off = align256(off + size_t(g.B) * (g.nreg > 0 ? g.nreg : 1));
  m.bfull = off;  off = align256(off + size_t(g.B) * g.nb);
  m.total = off;
  return m;
}

struct LayoutPtrs {
  int32_t* perm;     // [B, N] slot -> raster (| kPadFlag for pad)
  int32_t* iperm;    // [B, N] raster -> slot (| kPadFlag for pad)
  uint64_t* bmask;   // [B, nb] bit s: slot s of the block is a real token
  int32_t* bcount;   // [B, nb] number of real tokens in the block
  uint8_t* codes;    // [B, nreg] shape code per region
  uint8_t* bfull;    // [B, nb] 1 when all 64 slots of the block are real tokens
};

inline LayoutPtrs layout_ptrs(const Geo& g, void* buf) {
  LayoutMap m = layout_map(g);
  char* p = static_cast<char*>(buf);
  return {reinterpret_cast<int32_t*>(p + m.perm), reinterpret_cast<int32_t*>(p + m.iperm),
          reinterpret_cast<uint64_t*>(p + m.bmask), reinterpret_cast<int32_t*>(p + m.bcount),
          reinterpret_cast<uint8_t*>(p + m.codes), reinterpret_cast<uint8_t*>(p + m.bfull)};
}

// shape code -> (t, h, w) sides; code 0 is the 4x4x4 cube, codes 1..6 are
// (2,4,8) (2,8,4) (4,2,8) (4,8,2) (8,2,4) (8,4,2)
__host__ __device__ inline void shape_sides(int code, int& st, int& sh, int& sw) {
  if (code <= 0 || code > 6) {
    st = sh = sw = 4;
    return;
  }
  const int c = code - 1;          // 0..5
  st = 2 << (c / 2);               // 2,2,4,4,8,8
  const int lo = (c / 2 == 0) ? 4 : 2, hi = (c / 2 == 2) ? 4 : 8;
  // the two remaining sides are {lo, hi} in (h, w) order for even c, swapped for odd c
  sh = (c & 1) ? hi : lo;
  sw = (c & 1) ? lo : hi;
}

// Record a message for bsa_last_error() on the calling thread and return st.
bsa_status set_error(bsa_status st, const char* fmt, ...);

// ---- launchers (one per translation unit) -------------------------------
cudaError_t launch_layout(const Geo& g, const __nv_bfloat16* k, int64_t sb, int64_t sn,
                          int64_t sh, LayoutPtrs lp, cudaStream_t st);
cudaError_t launch_permute(const Geo& g, LayoutPtrs lp, const __nv_bfloat16* x, int64_t sb,
                           int64_t sn, int64_t sh, __nv_bfloat16* xp, cudaStream_t st);
cudaError_t launch_unpermute(const Geo& g, LayoutPtrs lp, const __nv_bfloat16* op,
                             __nv_bfloat16* o, int64_t sb, int64_t sn, int64_t sh,
                             cudaStream_t st);
cudaError_t launch_permute_pool(const Geo& g, LayoutPtrs lp, const __nv_bfloat16* q,
                                const __nv_bfloat16* k, const __nv_bfloat16* v, int64_t sb,
                                int64_t sn, int64_t sh, __nv_bfloat16* qp, __nv_bfloat16* kp,
                                __nv_bfloat16* vp, float* qpool, float* kpool, cudaStream_t st);
cudaError_t launch_pool(const Geo& g, LayoutPtrs lp, const __nv_bfloat16* qp,
                        const __nv_bfloat16* kp, float* qpool, float* kpool, cudaStream_t st);
// kmap (optional): 2-D map over the pooled keys [B*heads*nb rows, d] fp32,
// 32 x 256 boxes, 128-byte swizzle (the TMA-fed score tiles)
// status: where a bounded wait that runs out reports BSA_ERR_TIMEOUT
cudaError_t launch_select(const Geo& g, const float* qpool, const float* kpool, const float* gate,
                          const CUtensorMap* kmap, int32_t* idx, int32_t* cnt, int32_t* status,
                          cudaStream_t st);
cudaError_t launch_pool_raster(const Geo& g, LayoutPtrs lp, const __nv_bfloat16* q,
                               const __nv_bfloat16* k, int64_t sb, int64_t sn, int64_t sh,
                               float* qpool, float* kpool, cudaStream_t st);

// Pointers and strides of one attention launch.  Block order: q and o are
// permuted [B, heads, N, d] tensors (strides unused).  Raster order: q and o
// are raster [B, N, heads, d] tensors with element strides, addressed
// through the slot -> raster map `perm`.
struct AttnIO {
  const __nv_bfloat16* q;
  int64_t qsb, qsn, qsh;
  __nv_bfloat16* o;
  int64_t osb, osn, osh;
  const int32_t* perm;
  const uint8_t* codes;
  const uint64_t* bmask;
  const uint8_t* bfull;
  const int32_t* idx;
  const int32_t* cnt;
  int32_t* status;
  // window heads instead of index lists: int32 [heads][3] (w_t, w_y, w_x),
  // negative = unbounded; null for the list-driven walk
  const int32_t* windows;
  // optional output: per-row log-sum-exp (exp2 domain) [B, heads, N], block order
  float* lse;
};

// Pointers of one backward (block-order tensors [B, heads, N, d]).
struct BwdIO {
  const __nv_bfloat16 *q, *k, *v, *o, *dout;
  const float* lse;       // [B, heads, N] from the forward
  float* delta;           // workspace [B, heads, N]: rowsum(dO * O)
  uint32_t* kmask;        // workspace [B, heads, nb, ceil(nb/32)]: transposed lists
  const int32_t *idx, *cnt;
  const uint64_t* bmask;
  const uint8_t* bfull;
  __nv_bfloat16 *dq, *dk, *dv;
  int32_t* status;
};

// maps: K, V, Q, dO (3-D maps over the permuted tensors, 64-row boxes)
cudaError_t launch_attention_bwd(const Geo& g, const CUtensorMap* maps, const BwdIO& io,
                                 cudaStream_t st);

// TMA maps of K and V.  Block order: one 3-D map each over [B*heads, N, d].
// Raster order: [0] a 3-D map over [B, N, heads*d] for the prefix blocks
// (64 consecutive tokens), [1 + code] a 5-D map over [B, T, H, W, heads*d]
// whose box is one video block of shape code (0 = 4x4x4).
template <bool RASTER>
struct KVMaps;
template <>
struct KVMaps<false> {
  CUtensorMap k, v;
};
template <>
struct KVMaps<true> {
  CUtensorMap k[8], v[8];
};

cudaError_t launch_attention(const Geo& g, const KVMaps<false>& maps, const AttnIO& io,
                             bool dense, cudaStream_t st);
cudaError_t launch_attention_raster(const Geo& g, const KVMaps<true>& maps, const AttnIO& io,
                                    cudaStream_t st);

// ---- device helpers -----------------------------------------------------
#if defined(__CUDACC__)
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
// non-blocking probe of an mbarrier phase
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait on an mbarrier phase.  Gives up after `limit_ns` of wall
// time, or as soon as *abort (when not null) is set by another thread;
// returns false then.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                          uint64_t limit_ns = 2000000000ull) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63) == 0) {
      if (abort && *abort) return false;
      if (global_timer_ns() - t0 > limit_ns) return false;
    }
  }
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void tma_load_5d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2, int c3, int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
      "r"(c4)
      : "memory");
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ float4 ld_shared_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---- tcgen05 ---------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
// D[tmem] (+)= A[smem desc] * B[smem desc]
__device__ __forceinline__ void tc_mma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// UMMA shared-memory descriptor for a 128-byte-swizzled operand tile
// (sm_100 format: start>>4 in [0,14), LBO>>4 in [16,30), SBO>>4 in [32,46),
// version 1 in [46,48), layout type 2 = SWIZZLE_128B in [61,64)).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= uint64_t((saddr >> 4) & 0x3FFFu);
  d |= uint64_t((lbo >> 4) & 0x3FFFu) << 16;
  d |= uint64_t((sbo >> 4) & 0x3FFFu) << 32;
  d |= uint64_t(1) << 46;
  d |= uint64_t(2) << 61;
  return d;
}

// Instruction descriptor of kind::f16 with bf16 A/B, fp32 D, A K-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
         (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

#define BSA_TMEM_LD32(taddr, r)                                                                \
  asm volatile(                                                                                \
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "                                               \
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"                                \
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"          \
      "tcgen05.wait::ld.sync.aligned;"                                                         \
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),    \
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),             \
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),          \
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),          \
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),          \
        "=r"(r[31])                                                                            \
      : "r"(taddr)                                                                             \
      : "memory")

#define BSA_TMEM_ST32(taddr, r)                                                                \
  asm volatile(                                                                                \
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "                                         \
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"                               \
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n\t"                 \
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),                                           \
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),  \
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),        \
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),      \
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),      \
      "r"(r[29]), "r"(r[30]), "r"(r[31])                                                       \
      : "memory")

#define BSA_TMEM_LD64(taddr, r)  \
  asm volatile(  \
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n\t"  \
      "tcgen05.wait::ld.sync.aligned;"  \
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])  \
      : "r"(taddr)  \
      : "memory")

#define BSA_TMEM_ST64(taddr, r)  \
  asm volatile(  \
      "tcgen05.st.sync.aligned.32x32b.x64.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,%64};\n\t"  \
      "tcgen05.wait::st.sync.aligned;"  \
      :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31]), "r"(r[32]), "r"(r[33]), "r"(r[34]), "r"(r[35]), "r"(r[36]), "r"(r[37]), "r"(r[38]), "r"(r[39]), "r"(r[40]), "r"(r[41]), "r"(r[42]), "r"(r[43]), "r"(r[44]), "r"(r[45]), "r"(r[46]), "r"(r[47]), "r"(r[48]), "r"(r[49]), "r"(r[50]), "r"(r[51]), "r"(r[52]), "r"(r[53]), "r"(r[54]), "r"(r[55]), "r"(r[56]), "r"(r[57]), "r"(r[58]), "r"(r[59]), "r"(r[60]), "r"(r[61]), "r"(r[62]), "r"(r[63])  \
      : "memory")

// D[tmem] (+)= A[tmem] * B[smem desc]  (A read from tensor memory)
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// named barrier over a subset of the CTA's warps
__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two-lane fp32 arithmetic of sm_100 (one instruction for two independent
// lanes, each rounded exactly as the scalar instruction would round it).
__device__ __forceinline__ void fma_f32x2(float& y0, float& y1, float a0, float a1, float b0,
                                          float b1, float c0, float c1) {
  asm("{\n\t.reg .b64 a, b, c, d;\n\t"
      "mov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\tmov.b64 c, {%6, %7};\n\t"
      "fma.rn.f32x2 d, a, b, c;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(y0), "=f"(y1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
__device__ __forceinline__ void add_f32x2(float& y0, float& y1, float a0, float a1, float b0,
                                          float b1) {
  asm("{\n\t.reg .b64 a, b, d;\n\t"
      "mov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "add.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(y0), "=f"(y1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
// max of three (sm_100 three-input form)
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
#endif  // __CUDACC__

}  // namespace bsa
