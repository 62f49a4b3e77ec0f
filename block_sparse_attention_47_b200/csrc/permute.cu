// Token permutation between raster order and block order (Sparse VideoGen
// on TPU, aibase.it, section "실무에서 배울 최적화 기준": masks only become
// whole tiles once tokens are permuted).  Pure data movement, HBM-bound:
// every 16-byte vector is read once and written once.
//
// permute_kernel: consecutive threads take consecutive 16-byte vectors of
// one raster token row [heads, head_dim] (contiguous), so raster-side
// accesses are fully coalesced and block-order accesses are whole head_dim
// rows (128 or 256 contiguous bytes).  The fused permute + pool and the
// unpermute take one block of one head per CTA instead.
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

// Q, K and V moved to block order and the block means of Q and K taken from
// the rows as they pass (Prism / Kandinsky 6 speed ablation, oh-my-gpu.com,
// section "같은 계산량 안에서 볼 곳을 고르는 Prism": a block is judged by
// the mean of its 64 tokens), so the permuted Q and K are never read back.
// One CTA per (block, head, batch element); thread (rg, v) moves 16-byte
// channel vector v of rows rg, rg + G, .. and sums them in that order, then
// the row groups are added in order: the same order as the separate pooling
// kernels, so the means are bit-identical to theirs.
template <int D>
__global__ void __launch_bounds__(kThreads) permute_pool_kernel(
    Geo g, const int32_t* __restrict__ perm, const int32_t* __restrict__ bcount,
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const __nv_bfloat16* __restrict__ v, int64_t sb, int64_t sn, int64_t sh,
    __nv_bfloat16* __restrict__ qp, __nv_bfloat16* __restrict__ kp,
    __nv_bfloat16* __restrict__ vp, float* __restrict__ qpool, float* __restrict__ kpool) {
  constexpr int VEC = D / 8;               // 16-byte vectors per row
  constexpr int GROUPS = kThreads / VEC;   // row groups
  constexpr int RPT = kBlock / GROUPS;     // rows per thread
  const int j = blockIdx.x, hh = blockIdx.y, b = blockIdx.z;
  const int v8 = threadIdx.x % VEC, rg = threadIdx.x / VEC;
  __shared__ float red[2][GROUPS][D + 1];
  __shared__ int64_t src[kBlock];  // element offset of each slot's row, -1 for pad
  if (threadIdx.x < kBlock) {
    const uint32_t pr = uint32_t(perm[int64_t(b) * g.N + int64_t(j) * kBlock + threadIdx.x]);
    src[threadIdx.x] =
        (pr & kPad) ? -1 : int64_t(b) * sb + int64_t(pr) * sn + int64_t(hh) * sh;
  }
  __syncthreads();
  const int64_t dst0 = ((int64_t(b) * g.h + hh) * g.N + int64_t(j) * kBlock) * D + v8 * 8;
  int64_t off[RPT];
#pragma unroll
  for (int i = 0; i < RPT; ++i) off[i] = src[rg + GROUPS * i];
  // all rows of the three tensors in flight before any is stored
  uint4 val[3][RPT];
#pragma unroll
  for (int w = 0; w < 3; ++w) {
    const __nv_bfloat16* x = w == 0 ? q : (w == 1 ? k : v);
#pragma unroll
    for (int i = 0; i < RPT; ++i)
      val[w][i] = off[i] < 0 ? make_uint4(0, 0, 0, 0)
                             : *reinterpret_cast<const uint4*>(x + off[i] + v8 * 8);
  }
#pragma unroll
  for (int w = 0; w < 3; ++w) {
    __nv_bfloat16* xp = w == 0 ? qp : (w == 1 ? kp : vp);
#pragma unroll
    for (int i = 0; i < RPT; ++i)
      *reinterpret_cast<uint4*>(xp + dst0 + int64_t(rg + GROUPS * i) * D) = val[w][i];
  }
#pragma unroll
  for (int w = 0; w < 2; ++w) {
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
      if (off[i] < 0) continue;
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&val[w][i]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(p[e]);
        acc[2 * e] += f.x;
        acc[2 * e + 1] += f.y;
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) red[w][rg][v8 * 8 + e] = acc[e];
  }
  __syncthreads();
  const float inv = 1.0f / float(bcount[int64_t(b) * g.nb + j]);
  const int64_t out0 = ((int64_t(b) * g.h + hh) * g.nb + j) * D;
  for (int c = threadIdx.x; c < 2 * D; c += kThreads) {
    const int w = c / D, ch = c % D;
    float s = 0.f;
    for (int r = 0; r < GROUPS; ++r) s += red[w][r][ch];
    (w ? kpool : qpool)[out0 + ch] = s * inv;
  }
}

// Block order back to raster order, one CTA per (block, head, batch
// element): the block's 64 rows are read as one contiguous 16 KB (d = 128)
// run and each row is written to its token's place (a whole 256-byte
// segment); pad slots write zeros to their pad tokens, so every raster row
// is written once.
template <int D>
__global__ void __launch_bounds__(kThreads) unpermute_block_kernel(
    Geo g, const int32_t* __restrict__ perm, const __nv_bfloat16* __restrict__ op,
    __nv_bfloat16* __restrict__ o, int64_t sb, int64_t sn, int64_t sh) {
  constexpr int VEC = D / 8, GROUPS = kThreads / VEC, RPT = kBlock / GROUPS;
  const int j = blockIdx.x, hh = blockIdx.y, b = blockIdx.z;
  const int v8 = threadIdx.x % VEC, rg = threadIdx.x / VEC;
  const int64_t src0 = ((int64_t(b) * g.h + hh) * g.N + int64_t(j) * kBlock) * D + v8 * 8;
  uint4 val[RPT];
  uint32_t pr[RPT];
#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    const int slot = rg + GROUPS * i;
    pr[i] = uint32_t(__ldg(perm + int64_t(b) * g.N + int64_t(j) * kBlock + slot));
    val[i] = *reinterpret_cast<const uint4*>(op + src0 + int64_t(slot) * D);
  }
#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    const int64_t raster = int64_t(pr[i] & ~kPad);
    *reinterpret_cast<uint4*>(o + b * sb + raster * sn + hh * sh + v8 * 8) =
        (pr[i] & kPad) ? make_uint4(0, 0, 0, 0) : val[i];
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

cudaError_t launch_permute_pool(const Geo& g, LayoutPtrs lp, const __nv_bfloat16* q,
                                const __nv_bfloat16* k, const __nv_bfloat16* v, int64_t sb,
                                int64_t sn, int64_t sh, __nv_bfloat16* qp, __nv_bfloat16* kp,
                                __nv_bfloat16* vp, float* qpool, float* kpool, cudaStream_t st) {
  const dim3 grid(g.nb, g.h, g.B);
  if (g.d == 128)
    permute_pool_kernel<128><<<grid, kThreads, 0, st>>>(g, lp.perm, lp.bcount, q, k, v, sb, sn, sh,
                                                        qp, kp, vp, qpool, kpool);
  else
    permute_pool_kernel<64><<<grid, kThreads, 0, st>>>(g, lp.perm, lp.bcount, q, k, v, sb, sn, sh,
                                                       qp, kp, vp, qpool, kpool);
  return cudaGetLastError();
}

cudaError_t launch_unpermute(const Geo& g, LayoutPtrs lp, const __nv_bfloat16* op,
                             __nv_bfloat16* o, int64_t sb, int64_t sn, int64_t sh,
                             cudaStream_t st) {
  const dim3 grid(g.nb, g.h, g.B);
  if (g.d == 128)
    unpermute_block_kernel<128><<<grid, kThreads, 0, st>>>(g, lp.perm, op, o, sb, sn, sh);
  else
    unpermute_block_kernel<64><<<grid, kThreads, 0, st>>>(g, lp.perm, op, o, sb, sn, sh);
  return cudaGetLastError();
}

}  // namespace bsa
