// Block layout: which raster token sits in which 64-token block slot.
//
// Fixed mode: 4x4x4 cubes in (bt, bh, bw) raster order, tokens inside a cube
// in (t, y, x) raster order.  Dynamic mode: per (batch, 8x8x8 region) one of
// seven 64-token box shapes, chosen from the per-axis mean |delta K| with
// the short side on the most-changing axis (Prism / Kandinsky 6 speed
// ablation, oh-my-gpu.com, section "같은 계산량 안에서 볼 곳을 고르는
// Prism").  Both are HBM-bound: dynamic mode reads K once (plus neighbour
// re-reads served from L1/L2), the map build writes 8 bytes per token.
#include "bsa_internal.cuh"

namespace bsa {
namespace {

constexpr uint32_t kPad = 0x80000000u;

// ---- dynamic mode: per-region variation and shape code --------------------
// One CTA per (region, batch).  Work item = (y, x, 16-byte channel chunk);
// each item walks t and accumulates |delta| along t (previous t in
// registers), along y and x (neighbour token loaded, mostly from L1).
constexpr int kVarThreads = 256;

__device__ __forceinline__ float absdiff8(const uint4& a, const uint4& b) {
  const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a);
  const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b);
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 fa = __bfloat1622float2(pa[i]);
    float2 fb = __bfloat1622float2(pb[i]);
    s += fabsf(fa.x - fb.x) + fabsf(fa.y - fb.y);
  }
  return s;
}

__global__ void __launch_bounds__(kVarThreads) region_shape_kernel(
    Geo g, const __nv_bfloat16* __restrict__ k, int64_t sb, int64_t sn, int64_t sh,
    uint8_t* __restrict__ codes) {
  const int r = blockIdx.x, b = blockIdx.y;
  const int nrh = g.H / 8, nrw = g.W / 8;
  const int rt = r / (nrh * nrw), rem = r % (nrh * nrw);
  const int rh = rem / nrw, rw = rem % nrw;
  const int t0 = rt * 8, y0 = rh * 8, x0 = rw * 8;
  const int chunks_per_head = g.d / 8;
  const int chunks = g.h * chunks_per_head;
  const int items = 64 * chunks;

  float sum[3] = {0.f, 0.f, 0.f};
  int cnt[3] = {0, 0, 0};
  const __nv_bfloat16* kb = k + int64_t(b) * sb;

  for (int it = threadIdx.x; it < items; it += kVarThreads) {
    const int q = it % chunks;
    const int yx = it / chunks;
    const int yy = yx / 8, xx = yx % 8;
    const int hh = q / chunks_per_head, c0 = (q % chunks_per_head) * 8;
    const int y = y0 + yy, x = x0 + xx;
    const bool ok_y = y < g.Hv, ok_x = x < g.Wv;
    const bool ok_y1 = (yy < 7) && (y + 1 < g.Hv);
    const bool ok_x1 = (xx < 7) && (x + 1 < g.Wv);
    uint4 prev = make_uint4(0, 0, 0, 0);
    bool prev_ok = false;
    for (int tt = 0; tt < 8; ++tt) {
      const int t = t0 + tt;
      const bool ok = ok_y && ok_x && (t < g.Tv);
      const int64_t n = g.P + (int64_t(t) * g.H + y) * g.W + x;
      const uint4 cur = *reinterpret_cast<const uint4*>(kb + n * sn + int64_t(hh) * sh + c0);
      if (ok && prev_ok) {
        sum[0] += absdiff8(cur, prev);
        cnt[0] += 8;
      }
      if (ok && ok_y1) {
        const uint4 nb = *reinterpret_cast<const uint4*>(kb + (n + g.W) * sn + int64_t(hh) * sh + c0);
        sum[1] += absdiff8(nb, cur);
        cnt[1] += 8;
      }
      if (ok && ok_x1) {
        const uint4 nb = *reinterpret_cast<const uint4*>(kb + (n + 1) * sn + int64_t(hh) * sh + c0);
        sum[2] += absdiff8(nb, cur);
        cnt[2] += 8;
      }
      prev = cur;
      prev_ok = ok;
    }
  }

  __shared__ float s_sum[kVarThreads / 32][3];
  __shared__ int s_cnt[kVarThreads / 32][3];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int a = 0; a < 3; ++a) {
    float s = sum[a];
    int c = cnt[a];
    for (int o = 16; o > 0; o >>= 1) {
      s += __shfl_xor_sync(0xffffffffu, s, o);
      c += __shfl_xor_sync(0xffffffffu, c, o);
    }
    if (lane == 0) {
      s_sum[warp][a] = s;
      s_cnt[warp][a] = c;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float v[3];
    bool any_empty = false;
    for (int a = 0; a < 3; ++a) {
      float s = 0.f;
      long long c = 0;
      for (int w = 0; w < kVarThreads / 32; ++w) {
        s += s_sum[w][a];
        c += s_cnt[w][a];
      }
      any_empty |= (c == 0);
      v[a] = c ? s / float(c) : 0.f;
    }
    int code = 0;
    const float vmax = fmaxf(v[0], fmaxf(v[1], v[2]));
    const float vmin = fminf(v[0], fminf(v[1], v[2]));
    if (!any_empty && vmax > 0.f && !(vmax < g.tau * vmin)) {
      // rank axes by (v descending, axis ascending): sides 2, 4, 8
      int side[3];
      for (int a = 0; a < 3; ++a) {
        int rank = 0;
        for (int o = 0; o < 3; ++o)
          if (v[o] > v[a] || (v[o] == v[a] && o < a)) ++rank;
        side[a] = 2 << rank;
      }
      for (int c = 1; c < 7; ++c) {
        int st, shh, sw;
        shape_sides(c, st, shh, sw);
        if (st == side[0] && shh == side[1] && sw == side[2]) code = c;
      }
    }
    codes[int64_t(b) * g.nreg + r] = uint8_t(code);
  }
}

// ---- slot <-> raster maps -------------------------------------------------
// One CTA of 64 threads per (block, batch): thread s owns slot s.
__global__ void __launch_bounds__(64) build_maps_kernel(Geo g, const uint8_t* __restrict__ codes,
                                                        int32_t* __restrict__ perm,
                                                        int32_t* __restrict__ iperm,
                                                        uint64_t* __restrict__ bmask,
                                                        int32_t* __restrict__ bcount,
                                                        uint8_t* __restrict__ bfull) {
  const int j = blockIdx.x, b = blockIdx.y, s = threadIdx.x;
  const int slot = j * kBlock + s;
  int raster;
  bool valid;
  if (j < g.nbp) {
    raster = slot;
    valid = false;
    for (int i = 0; i < g.nseg; ++i)
      if (slot >= g.seg_off[i] && slot < g.seg_off[i] + g.seg_len[i]) valid = true;
  } else {
    const int jv = j - g.nbp;
    int t, y, x;
    if (g.mode == BSA_BLOCK_FIXED_444) {
      const int nbh = g.H / 4, nbw = g.W / 4;
      const int bt = jv / (nbh * nbw), rem = jv % (nbh * nbw);
      const int bh = rem / nbw, bw = rem % nbw;
      t = 4 * bt + s / 16;
      y = 4 * bh + (s / 4) % 4;
      x = 4 * bw + s % 4;
    } else {
      const int r = jv / 8, sub = jv % 8;
      const int nrh = g.H / 8, nrw = g.W / 8;
      const int rt = r / (nrh * nrw), rem = r % (nrh * nrw);
      const int rh = rem / nrw, rw = rem % nrw;
      int st, sh, sw;
      shape_sides(codes[int64_t(b) * g.nreg + r], st, sh, sw);
      const int gh = 8 / sh, gw = 8 / sw;
      const int bt = sub / (gh * gw), bh = (sub / gw) % gh, bw = sub % gw;
      t = 8 * rt + st * bt + s / (sh * sw);
      y = 8 * rh + sh * bh + (s / sw) % sh;
      x = 8 * rw + sw * bw + s % sw;
    }
    raster = g.P + (t * g.H + y) * g.W + x;
    valid = (t < g.Tv) && (y < g.Hv) && (x < g.Wv);
  }
  const int64_t base = int64_t(b) * g.N;
  const uint32_t flag = valid ? 0u : kPad;
  perm[base + slot] = int32_t(uint32_t(raster) | flag);
  iperm[base + raster] = int32_t(uint32_t(slot) | flag);
  const uint32_t bal = __ballot_sync(0xffffffffu, valid);
  __shared__ uint32_t s_bal[2];
  if ((s & 31) == 0) s_bal[s >> 5] = bal;
  __syncthreads();
  if (s == 0) {
    const uint64_t m = uint64_t(s_bal[0]) | (uint64_t(s_bal[1]) << 32);
    bmask[int64_t(b) * g.nb + j] = m;
    bcount[int64_t(b) * g.nb + j] = __popcll(m);
    bfull[int64_t(b) * g.nb + j] = (m == ~0ull) ? 1 : 0;
  }
}

}  // namespace

cudaError_t launch_layout(const Geo& g, const __nv_bfloat16* k, int64_t sb, int64_t sn,
                          int64_t sh, LayoutPtrs lp, cudaStream_t st) {
  if (g.mode == BSA_BLOCK_DYNAMIC_888) {
    region_shape_kernel<<<dim3(g.nreg, g.B), kVarThreads, 0, st>>>(g, k, sb, sn, sh, lp.codes);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  build_maps_kernel<<<dim3(g.nb, g.B), 64, 0, st>>>(g, lp.codes, lp.perm, lp.iperm, lp.bmask,
                                                    lp.bcount, lp.bfull);
  return cudaGetLastError();
}

}  // namespace bsa
