// Token permutation between raster order and block order (Sparse VideoGen
// on TPU, aibase.it, section "실무에서 배울 최적화 기준": masks only become
// whole tiles once tokens are permuted).  Pure data movement, HBM-bound:
// every 16-byte vector is read once and written once.
//
// Thread mapping: consecutive threads take consecutive 16-byte vectors of
// one raster token row [heads, head_dim] (contiguous), so raster-side
// accesses are fully coalesced and block-order accesses are whole
// head_dim rows (128 or 256 contiguous bytes).
#include "bsa_internal.cuh"

namespace bsa {
namespace {

constexpr uint32_t kPad = 0x80000000u;
constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads) permute_kernel(
    Geo g, const int32_t* __restrict__ perm, const __nv_bfloat16* __restrict__ x, int64_t sb,
    int64_t sn, int64_t sh, __nv_bfloat16* __restrict__ xp) {
  const int vec_per_row = g.d / 8;
  const int64_t per_token = int64_t(g.h) * vec_per_row;
  const int64_t total = int64_t(g.B) * g.N * per_token;
  for (int64_t i = blockIdx.x * int64_t(kThreads) + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * kThreads) {
    const int v = int(i % vec_per_row);
    const int64_t rest = i / vec_per_row;
    const int hh = int(rest % g.h);
    const int64_t bs = rest / g.h;  // b * N + slot
    const int b = int(bs / g.N);
    const int slot = int(bs % g.N);
    const uint32_t pr = uint32_t(perm[bs]);
    uint4 val = make_uint4(0, 0, 0, 0);
    if (!(pr & kPad)) {
      const int raster = int(pr);
      val = *reinterpret_cast<const uint4*>(x + b * sb + raster * sn + hh * sh + v * 8);
    }
    __nv_bfloat16* dst = xp + ((int64_t(b) * g.h + hh) * g.N + slot) * g.d + v * 8;
    *reinterpret_cast<uint4*>(dst) = val;
  }
}

__global__ void __launch_bounds__(kThreads) unpermute_kernel(
    Geo g, const int32_t* __restrict__ iperm, const __nv_bfloat16* __restrict__ op,
    __nv_bfloat16* __restrict__ o, int64_t sb, int64_t sn, int64_t sh) {
  const int vec_per_row = g.d / 8;
  const int64_t per_token = int64_t(g.h) * vec_per_row;
  const int64_t total = int64_t(g.B) * g.N * per_token;
  for (int64_t i = blockIdx.x * int64_t(kThreads) + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * kThreads) {
    const int v = int(i % vec_per_row);
    const int64_t rest = i / vec_per_row;
    const int hh = int(rest % g.h);
    const int64_t bn = rest / g.h;  // b * N + raster
    const int b = int(bn / g.N);
    const int raster = int(bn % g.N);
    const uint32_t is = uint32_t(iperm[bn]);
    uint4 val = make_uint4(0, 0, 0, 0);
    if (!(is & kPad)) {
      const int slot = int(is);
      val = *reinterpret_cast<const uint4*>(op + ((int64_t(b) * g.h + hh) * g.N + slot) * g.d +
                                            v * 8);
    }
    *reinterpret_cast<uint4*>(o + b * sb + raster * sn + hh * sh + v * 8) = val;
  }
}

int grid_for(int64_t work) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (work + kThreads - 1) / kThreads;
  const int64_t cap = int64_t(sms) * 8;  // 8 resident CTAs of 256 threads per SM
  return int(want < cap ? want : cap);
}

}  // namespace

cudaError_t launch_permute(const Geo& g, LayoutPtrs lp, const __nv_bfloat16* x, int64_t sb,
                           int64_t sn, int64_t sh, __nv_bfloat16* xp, cudaStream_t st) {
  const int64_t work = int64_t(g.B) * g.N * g.h * (g.d / 8);
  permute_kernel<<<grid_for(work), kThreads, 0, st>>>(g, lp.perm, x, sb, sn, sh, xp);
  return cudaGetLastError();
}

cudaError_t launch_unpermute(const Geo& g, LayoutPtrs lp, const __nv_bfloat16* op,
                             __nv_bfloat16* o, int64_t sb, int64_t sn, int64_t sh,
                             cudaStream_t st) {
  const int64_t work = int64_t(g.B) * g.N * g.h * (g.d / 8);
  unpermute_kernel<<<grid_for(work), kThreads, 0, st>>>(g, lp.iperm, op, o, sb, sn, sh);
  return cudaGetLastError();
}

}  // namespace bsa
