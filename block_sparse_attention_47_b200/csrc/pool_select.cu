// Block mean pooling and top-k key-block selection.
//
// Pooling (Prism / Kandinsky 6 speed ablation, oh-my-gpu.com, section
// "같은 계산량 안에서 볼 곳을 고르는 Prism": a block is judged by the mean of
// its 64 tokens): pad slots are zero in block order, so the mean is the sum
// of the 64 rows divided by the block's valid count.  HBM-bound.
//
// Selection (same section: keep the most relevant key blocks, 25 % at
// sparsity 0.75; Ref2VA VSA, pulmap.app, section "조건 토큰은 왜 다르게
// 다루나": the conditioning prefix is always kept and top-k runs over video
// key blocks only).  Scores are fp32 dot products of the pooled means; the
// k-th largest is found by an exact 4-pass radix select on order-preserving
// 32-bit keys, then a warp compacts the winners in ascending index order, so
// ties at the threshold go to the lowest indices and the list comes out
// sorted.  The score matrix never leaves shared memory.
#include "bsa_internal.cuh"

namespace bsa {
namespace {

// ---- pooling --------------------------------------------------------------
// One CTA per (block, head, batch) for both Q and K: thread (r, v) sums rows
// r, r+16, r+32, r+48 of 16-byte channel vector v, then a shared reduction.
constexpr int kPoolThreads = 256;

__global__ void __launch_bounds__(kPoolThreads) pool_kernel(
    Geo g, const int32_t* __restrict__ bcount, const __nv_bfloat16* __restrict__ qp,
    const __nv_bfloat16* __restrict__ kp, float* __restrict__ qpool, float* __restrict__ kpool) {
  const int j = blockIdx.x, hh = blockIdx.y, b = blockIdx.z;
  const int vec = g.d / 8;            // 16 (d=128) or 8 (d=64)
  const int groups = kPoolThreads / vec;  // row groups
  const int v = threadIdx.x % vec, rg = threadIdx.x / vec;
  const int64_t row0 = (int64_t(b) * g.h + hh) * g.N + int64_t(j) * kBlock;
  __shared__ float red[2][kPoolThreads / 8][129];
  for (int which = 0; which < 2; ++which) {
    const __nv_bfloat16* x = which ? kp : qp;
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int r = rg; r < kBlock; r += groups) {
      const uint4 u = *reinterpret_cast<const uint4*>(x + (row0 + r) * g.d + v * 8);
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float2 f = __bfloat1622float2(p[i]);
        acc[2 * i] += f.x;
        acc[2 * i + 1] += f.y;
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) red[which][rg][v * 8 + i] = acc[i];
  }
  __syncthreads();
  const float inv = 1.0f / float(bcount[int64_t(b) * g.nb + j]);
  const int64_t out0 = ((int64_t(b) * g.h + hh) * g.nb + j) * g.d;
  for (int c = threadIdx.x; c < 2 * g.d; c += kPoolThreads) {
    const int which = c / g.d, ch = c % g.d;
    float s = 0.f;
    for (int r = 0; r < groups; ++r) s += red[which][r][ch];
    (which ? kpool : qpool)[out0 + ch] = s * inv;
  }
}

// The same block means read straight from raster Q and K through the
// layout's slot -> raster map (no permuted copies).  Rows are summed in the
// same order as pool_kernel (pad slots, zero there, are skipped here), so
// the two give bit-identical means.
__global__ void __launch_bounds__(kPoolThreads) pool_raster_kernel(
    Geo g, const int32_t* __restrict__ perm, const int32_t* __restrict__ bcount,
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k, int64_t sb,
    int64_t sn, int64_t sh, float* __restrict__ qpool, float* __restrict__ kpool) {
  const int j = blockIdx.x, hh = blockIdx.y, b = blockIdx.z;
  const int vec = g.d / 8;
  const int groups = kPoolThreads / vec;
  const int v = threadIdx.x % vec, rg = threadIdx.x / vec;
  __shared__ float red[2][kPoolThreads / 8][129];
  __shared__ int64_t src[kBlock];  // element offset of each slot's row, -1 for pad
  if (threadIdx.x < kBlock) {
    const uint32_t pr = uint32_t(perm[int64_t(b) * g.N + int64_t(j) * kBlock + threadIdx.x]);
    src[threadIdx.x] =
        (pr & 0x80000000u) ? -1 : int64_t(b) * sb + int64_t(pr) * sn + int64_t(hh) * sh;
  }
  __syncthreads();
  for (int which = 0; which < 2; ++which) {
    const __nv_bfloat16* x = which ? k : q;
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int r = rg; r < kBlock; r += groups) {
      const int64_t off = src[r];
      if (off < 0) continue;
      const uint4 u = *reinterpret_cast<const uint4*>(x + off + v * 8);
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float2 f = __bfloat1622float2(p[i]);
        acc[2 * i] += f.x;
        acc[2 * i + 1] += f.y;
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) red[which][rg][v * 8 + i] = acc[i];
  }
  __syncthreads();
  const float inv = 1.0f / float(bcount[int64_t(b) * g.nb + j]);
  const int64_t out0 = ((int64_t(b) * g.h + hh) * g.nb + j) * g.d;
  for (int c = threadIdx.x; c < 2 * g.d; c += kPoolThreads) {
    const int which = c / g.d, ch = c % g.d;
    float s = 0.f;
    for (int r = 0; r < groups; ++r) s += red[which][r][ch];
    (which ? kpool : qpool)[out0 + ch] = s * inv;
  }
}

// ---- selection --------------------------------------------------------------
// A CTA scores kSelRows query blocks per row group of kSelThreads threads
// (RG groups share every staged key chunk) and then takes one query block
// per warp in the top-k phase.
constexpr int kSelThreads = 256;
constexpr int kSelRows = 8;

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t u) {
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u);
}

// One 256-bin radix pass of the top-k over a row's keys: counts the keys
// that pass `in_set` by `digit_of`, then finds the digit D holding the
// want-th largest (count(digit > D) < want <= count(digit >= D)); returns D,
// lowers `want` by count(digit > D) and sets `at` to count(digit == D).
template <class InSet, class DigitOf>
__device__ __forceinline__ int radix_pass(const uint32_t* key, int nbv, uint32_t* hist, int lane,
                                          int& want, int& at, InSet in_set, DigitOf digit_of) {
  for (int i = lane; i < 256; i += 32) hist[i] = 0;
  __syncwarp();
  // eight keys in flight per lane before their histogram updates
  for (int base = 0; base < nbv; base += 8 * 32) {
    uint32_t u[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int jv = base + 32 * i + lane;
      u[i] = jv < nbv ? key[jv] : 0u;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (base + 32 * i + lane < nbv && in_set(u[i])) atomicAdd(&hist[digit_of(u[i])], 1u);
  }
  __syncwarp();
  // lane l owns digits [8*(31-l), 8*(31-l)+8), scanned from the top
  uint32_t local[8];
  uint32_t tot = 0;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    local[q] = hist[8 * (31 - lane) + (7 - q)];  // descending digits
    tot += local[q];
  }
  uint32_t incl = tot;  // inclusive prefix over lanes (higher digits first)
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  const uint32_t excl = incl - tot;
  const bool mine = (excl < uint32_t(want)) && (incl >= uint32_t(want));
  const uint32_t who = __ballot_sync(0xffffffffu, mine);
  const int src = __ffs(who) - 1;
  int digit = 0, above = 0, here = 0;
  if (mine) {
    uint32_t run = excl;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      if (run + local[q] >= uint32_t(want)) {
        digit = 8 * (31 - lane) + (7 - q);
        above = int(run);
        here = int(local[q]);
        break;
      }
      run += local[q];
    }
  }
  digit = __shfl_sync(0xffffffffu, digit, src);
  above = __shfl_sync(0xffffffffu, above, src);
  at = __shfl_sync(0xffffffffu, here, src);
  want -= above;
  __syncwarp();
  return digit;
}

// The smallest key u in [lo, hi) with pred(u) (pred monotone: false then
// true), or hi when there is none; 32 probes per step, so a 32-bit range
// takes at most eight steps (twelve are allowed).
template <class Pred>
__device__ __forceinline__ uint64_t first_key_where(uint64_t lo, uint64_t hi, int lane, Pred pred) {
  for (int it = 0; it < 12 && lo < hi; ++it) {
    const uint64_t span = hi - lo;
    const uint64_t p = lo + (span * uint64_t(lane)) / 32u;
    const uint32_t b = __ballot_sync(0xffffffffu, pred(uint32_t(p)));
    if (b == 0u) {
      lo = __shfl_sync(0xffffffffu, p, 31) + 1u;
    } else {
      const int l = __ffs(b) - 1;
      const uint64_t at = __shfl_sync(0xffffffffu, p, l);
      const uint64_t before = __shfl_sync(0xffffffffu, p, l > 0 ? l - 1 : 0);
      hi = at;
      if (l > 0) lo = before + 1u;
    }
  }
  return hi;
}

// Score tiles: KPT key blocks per thread, so kSelThreads * KPT pooled key
// rows per pass, staged through shared memory 32 channels at a time with
// coalesced 16-byte loads (row stride 36 floats: the 16-byte reads of 8
// consecutive rows hit 8 distinct bank quads).
constexpr int kSelChunk = 32;
constexpr int kSelStride = kSelChunk + 4;
// the TMA form stages 16 channels (one 64-byte row) of 256 * KPT pooled keys
// per chunk
constexpr int kSelChunkTma = 16;

template <int KPT>
constexpr size_t select_tile_floats() {
  return size_t(kSelThreads) * KPT * kSelStride;
}

// dynamic smem: q rows [ROWS][d] fp32, keys [ROWS][nbv] u32, then the key
// tile (KPT > 0), whose space the histograms [ROWS warps][256] u32 of the
// top-k phase reuse.  ROWS = 8 * RG query blocks, NT = 256 * RG threads:
// thread t takes key slot t % 256 (+ 256 u) for the 8 rows of group t / 256.
//
// KPT > 0: every score is one fmaf chain over the channels in ascending
// order, as in the KPT == 0 form (one key block per thread read straight
// from global memory, for sequences whose scores leave no room for a tile),
// so both give bit-identical lists.
//
// gate (optional, fp32 [heads][d][d]): the learned-gate score of the VSA
// description (Ref2VA VSA, pulmap.app, section "토큰 75%를 건너뛰는 VSA": a
// trained predictor, to_gate_compress, decides which tiles matter): each
// pooled query row is first mapped through its head's gate matrix,
// q~_c = sum_e G[c][e] q_e (one fmaf chain in e order), and the key blocks
// are scored against q~.  G = identity gives the ungated scores bit for bit.
template <int KPT, bool TMA, int RG>
__global__ void __launch_bounds__(kSelThreads * RG) select_kernel(
    const __grid_constant__ CUtensorMap kmap, Geo g, const float* __restrict__ qpool,
    const float* __restrict__ kpool, const float* __restrict__ gate, int32_t* __restrict__ idx,
    int32_t* __restrict__ cnt) {
  constexpr int NT = kSelThreads * RG, ROWS = kSelRows * RG;
  extern __shared__ __align__(16) unsigned char smem[];
  float* sq = reinterpret_cast<float*>(smem);
  uint32_t* skey = reinterpret_cast<uint32_t*>(sq + ROWS * g.d);
  float* stile = reinterpret_cast<float*>(skey + ((ROWS * g.nbv + 3) & ~3));
  uint32_t* shist = KPT > 0 ? reinterpret_cast<uint32_t*>(stile) : skey + ROWS * g.nbv;

  const int bh = blockIdx.y;
  const int i0 = blockIdx.x * ROWS;  // first video query block of this CTA
  const int rows = min(ROWS, g.nbv - i0);
  const int64_t pool0 = int64_t(bh) * g.nb * g.d;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kt = threadIdx.x % kSelThreads;  // key slot
  const float* sqg = sq + (threadIdx.x / kSelThreads) * kSelRows * g.d;  // this group's rows
  uint32_t* skeyg = skey + (threadIdx.x / kSelThreads) * kSelRows * g.nbv;

  // prefix query blocks attend densely: mark them once per (b, h)
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < g.nbp; i += NT) cnt[int64_t(bh) * g.nb + i] = -1;

  for (int e = threadIdx.x; e < ROWS * g.d; e += NT) {
    const int r = e / g.d, c = e % g.d;
    sq[e] = r < rows ? qpool[pool0 + int64_t(g.nbp + i0 + r) * g.d + c] : 0.f;
  }
  __syncthreads();
  if (gate) {
    // q~ = G q for every row: thread t takes channel c = t % d of rows t / d,
    // t / d + NT / d, .. (NT is a multiple of d), so each thread reads row c
    // of G once for all its outputs; each output is one fmaf chain in e order
    const float* G = gate + int64_t(bh % g.h) * g.d * g.d;
    constexpr int MAXO = (ROWS * 128) / NT;  // outputs per thread at d = 128
    const int c = threadIdx.x % g.d, r0 = threadIdx.x / g.d, rstep = NT / g.d;
    const int nout = ROWS * g.d / NT;
    float acc[MAXO];
#pragma unroll
    for (int o = 0; o < MAXO; ++o) acc[o] = 0.f;
    const float4* gr = reinterpret_cast<const float4*>(G + int64_t(c) * g.d);
    for (int e4 = 0; e4 < g.d / 4; ++e4) {
      const float4 gv = __ldg(gr + e4);
#pragma unroll
      for (int o = 0; o < MAXO; ++o) {
        if (o < nout) {
          const float4 qv = reinterpret_cast<const float4*>(sq + (r0 + rstep * o) * g.d)[e4];
          acc[o] = fmaf(gv.x, qv.x, acc[o]);
          acc[o] = fmaf(gv.y, qv.y, acc[o]);
          acc[o] = fmaf(gv.z, qv.z, acc[o]);
          acc[o] = fmaf(gv.w, qv.w, acc[o]);
        }
      }
    }
    __syncthreads();
#pragma unroll
    for (int o = 0; o < MAXO; ++o)
      if (o < nout) sq[(r0 + rstep * o) * g.d + c] = acc[o];
    __syncthreads();
  }

  if constexpr (TMA) {
    // scores, register-tiled as below, with the pooled-key chunks (KT rows x
    // 16 channels, 64-byte rows) brought in by TMA into two 64-byte-swizzled
    // buffers: the next chunk's copy runs while this one is multiplied.  A
    // chunk is 64-row boxes spread over the warps (one thread keeps only ~25
    // bytes per cycle of bulk copies in flight).  Each thread holds a
    // channel quad of its 8 query rows in registers and sweeps its KPT keys
    // with it: 8 broadcast and KPT 512-byte shared loads per 32 KPT FMAs.
    constexpr int CH = kSelChunkTma;
    constexpr int KT = kSelThreads * KPT;
    constexpr int TILE = KT * CH * 4;
    constexpr int PARTS = KT / 64;
    constexpr int ISSUERS = PARTS < NT / 32 ? PARTS : NT / 32;
    static_assert(PARTS % ISSUERS == 0, "whole boxes per issuing warp");
    const uint32_t tiles = (smem_u32(stile) + 1023u) & ~1023u;
    const uint32_t bar = tiles + 2 * TILE;
    const int ncpp = g.d / CH;                            // chunks per pass
    const int total = ((g.nbv + KT - 1) / KT) * ncpp;
    const int row0 = bh * g.nb + g.nbp;                   // this (b, h)'s first video key row
    if (threadIdx.x == 0) {
      mbar_init(bar, ISSUERS);
      mbar_init(bar + 8, ISSUERS);
      fence_mbar_init();
    }
    __syncthreads();
    // lane 0 of warp w < ISSUERS: boxes w, w + ISSUERS, .. of chunk c
    const bool issuer = lane == 0 && warp < ISSUERS;
    auto issue = [&](int c) {
      const int kb = (c / ncpp) * KT, cc = (c % ncpp) * CH;
      const uint32_t b8 = bar + 8u * uint32_t(c & 1);
      mbar_arrive_expect_tx(b8, TILE / ISSUERS);
      for (int part = warp; part < PARTS; part += ISSUERS)
        tma_load_2d(tiles + (c & 1) * TILE + part * 64 * CH * 4, &kmap, b8, cc,
                    row0 + kb + part * 64);
    };
    if (issuer) issue(0);
    float acc[kSelRows][KPT];
    for (int c = 0; c < total; ++c) {
      // buffer (c+1)&1 was last read in chunk c-1, which ended in a barrier
      if (issuer && c + 1 < total) issue(c + 1);
      const int kb = (c / ncpp) * KT, cc = (c % ncpp) * CH;
      if (cc == 0) {
#pragma unroll
        for (int r = 0; r < kSelRows; ++r)
#pragma unroll
          for (int u = 0; u < KPT; ++u) acc[r][u] = 0.f;
      }
      mbar_wait(bar + 8u * uint32_t(c & 1), (c >> 1) & 1, nullptr);
      const uint32_t buf = tiles + (c & 1) * TILE;
#pragma unroll
      for (int c4 = 0; c4 < CH / 4; ++c4) {
        float4 kv[KPT];
#pragma unroll
        for (int u = 0; u < KPT; ++u) {
          // 64-byte swizzle: 16-byte unit c4 of row rr sits at c4 ^ ((rr >> 1) & 3)
          const int rr = kt + kSelThreads * u;
          kv[u] = ld_shared_f4(buf + rr * 64 + ((c4 ^ ((rr >> 1) & 3)) << 4));
        }
        float4 qv[kSelRows];
#pragma unroll
        for (int r = 0; r < kSelRows; ++r)
          qv[r] = *reinterpret_cast<const float4*>(sqg + r * g.d + cc + 4 * c4);
        // component-major, so that 8*KPT independent chains sit between two
        // dependent FMAs (each chain still adds channels in ascending order)
#pragma unroll
        for (int r = 0; r < kSelRows; ++r)
#pragma unroll
          for (int u = 0; u < KPT; ++u) acc[r][u] = fmaf(qv[r].x, kv[u].x, acc[r][u]);
#pragma unroll
        for (int r = 0; r < kSelRows; ++r)
#pragma unroll
          for (int u = 0; u < KPT; ++u) acc[r][u] = fmaf(qv[r].y, kv[u].y, acc[r][u]);
#pragma unroll
        for (int r = 0; r < kSelRows; ++r)
#pragma unroll
          for (int u = 0; u < KPT; ++u) acc[r][u] = fmaf(qv[r].z, kv[u].z, acc[r][u]);
#pragma unroll
        for (int r = 0; r < kSelRows; ++r)
#pragma unroll
          for (int u = 0; u < KPT; ++u) acc[r][u] = fmaf(qv[r].w, kv[u].w, acc[r][u]);
      }
      if (cc + CH == g.d) {
#pragma unroll
        for (int u = 0; u < KPT; ++u) {
          const int jv = kb + kt + kSelThreads * u;
          if (jv < g.nbv)
#pragma unroll
            for (int r = 0; r < kSelRows; ++r) skeyg[r * g.nbv + jv] = order_key(acc[r][u]);
        }
      }
      __syncthreads();
    }
  } else if constexpr (KPT > 0) {
    static_assert(RG == 1, "one row group without TMA");
    // scores, register-tiled: thread t owns key blocks kb + t + 256*u
    // (u < KPT) for all 8 rows
    constexpr int KT = kSelThreads * KPT;
    const float* kbase = kpool + pool0 + int64_t(g.nbp) * g.d;
    for (int kb = 0; kb < g.nbv; kb += KT) {
      float acc[kSelRows][KPT];
#pragma unroll
      for (int r = 0; r < kSelRows; ++r)
#pragma unroll
        for (int u = 0; u < KPT; ++u) acc[r][u] = 0.f;
      for (int cc = 0; cc < g.d; cc += kSelChunk) {
        __syncthreads();  // the previous chunk has been read
        // rows kb..kb+KT-1, channels cc..cc+31: 8 float4 per row, coalesced
        for (int e = threadIdx.x; e < KT * (kSelChunk / 4); e += kSelThreads) {
          const int kr = e >> 3, c4 = e & 7;
          float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
          if (kb + kr < g.nbv)
            val = __ldg(reinterpret_cast<const float4*>(kbase + int64_t(kb + kr) * g.d + cc) + c4);
          *reinterpret_cast<float4*>(stile + kr * kSelStride + 4 * c4) = val;
        }
        __syncthreads();
#pragma unroll
        for (int c4 = 0; c4 < kSelChunk / 4; ++c4) {
          float4 kv[KPT];
#pragma unroll
          for (int u = 0; u < KPT; ++u)
            kv[u] = *reinterpret_cast<const float4*>(stile + (threadIdx.x + kSelThreads * u) *
                                                                 kSelStride + 4 * c4);
#pragma unroll
          for (int r = 0; r < kSelRows; ++r) {
            const float4 qv = *reinterpret_cast<const float4*>(sq + r * g.d + cc + 4 * c4);
#pragma unroll
            for (int u = 0; u < KPT; ++u) {
              acc[r][u] = fmaf(qv.x, kv[u].x, acc[r][u]);
              acc[r][u] = fmaf(qv.y, kv[u].y, acc[r][u]);
              acc[r][u] = fmaf(qv.z, kv[u].z, acc[r][u]);
              acc[r][u] = fmaf(qv.w, kv[u].w, acc[r][u]);
            }
          }
        }
      }
#pragma unroll
      for (int u = 0; u < KPT; ++u) {
        const int jv = kb + threadIdx.x + kSelThreads * u;
        if (jv < g.nbv)
#pragma unroll
          for (int r = 0; r < kSelRows; ++r) skey[r * g.nbv + jv] = order_key(acc[r][u]);
      }
    }
  } else
  // scores: thread per key block, all rows of the CTA at once
  for (int jv = threadIdx.x; jv < g.nbv; jv += kSelThreads) {
    const float4* kr = reinterpret_cast<const float4*>(kpool + pool0 + int64_t(g.nbp + jv) * g.d);
    float acc[kSelRows];
#pragma unroll
    for (int r = 0; r < kSelRows; ++r) acc[r] = 0.f;
    for (int c4 = 0; c4 < g.d / 4; ++c4) {
      const float4 kv = __ldg(kr + c4);
#pragma unroll
      for (int r = 0; r < kSelRows; ++r) {
        const float4 qv = reinterpret_cast<const float4*>(sq + r * g.d)[c4];
        acc[r] = fmaf(qv.x, kv.x, acc[r]);
        acc[r] = fmaf(qv.y, kv.y, acc[r]);
        acc[r] = fmaf(qv.z, kv.z, acc[r]);
        acc[r] = fmaf(qv.w, kv.w, acc[r]);
      }
    }
#pragma unroll
    for (int r = 0; r < kSelRows; ++r) skey[r * g.nbv + jv] = order_key(acc[r]);
  }
  __syncthreads();

  // top-k: one warp per query row
  if (warp < rows) {
    const uint32_t* key = skey + warp * g.nbv;
    uint32_t* hist = shist + warp * 256;
    // First pass: 256 bins linear in the score value between the row's
    // minimum and maximum (monotone in the key).  The top bits of float keys
    // fall in a handful of bins (one per binade), which would serialise the
    // histogram's atomics; value-linear bins spread them.  Then the usual
    // four 8-bit passes over the keys, restricted to the chosen bin.
    uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
    for (int jv = lane; jv < g.nbv; jv += 32) {
      const uint32_t u = key[jv];
      kmin = min(kmin, u);
      kmax = max(kmax, u);
    }
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    const float fmin = key_value(kmin), fmax = key_value(kmax);
    float scale = 256.f / (fmax - fmin);
    if (!(scale < 3.0e38f)) scale = 0.f;  // equal or non-finite range: one bin
    auto bin_of = [&](uint32_t u) {
      return int(fminf((key_value(u) - fmin) * scale, 255.f));
    };
    int want = g.keep, at = 0;
    const int vbin =
        radix_pass(key, g.nbv, hist, lane, want, at, [](uint32_t) { return true; }, bin_of);
    const uint32_t below = (1u << lane) - 1u;
    // the bin is a contiguous key range [blo, bhi): bins grow with the key
    const uint64_t kend = uint64_t(kmax) + 1u;
    const uint64_t blo =
        first_key_where(kmin, kend, lane, [&](uint32_t u) { return bin_of(u) >= vbin; });
    const uint64_t bhi =
        first_key_where(blo, kend, lane, [&](uint32_t u) { return bin_of(u) > vbin; });
    auto in_bin = [&](uint32_t u) { return uint64_t(u) >= blo && uint64_t(u) < bhi; };
    // the keys of that bin, gathered into a short list when they fit (the
    // staging space after the histograms holds CAND keys per warp)
    constexpr int CAND = KPT > 0 ? 512 : 0;
    uint32_t* cand = shist + ROWS * 256 + warp * CAND;
    int ncand = 0;
    if constexpr (CAND > 0) {
      for (int base = 0; base < g.nbv; base += 4 * 32) {
        uint32_t u[4];
        bool in[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int jv = base + 32 * i + lane;
          u[i] = jv < g.nbv ? key[jv] : 0u;
          in[i] = jv < g.nbv && in_bin(u[i]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t bal = __ballot_sync(0xffffffffu, in[i]);
          const int pos = ncand + __popc(bal & below);
          if (in[i] && pos < CAND) cand[pos] = u[i];
          ncand += __popc(bal);
        }
      }
      __syncwarp();
    }
    const bool short_list = CAND > 0 && ncand <= CAND;
    uint32_t prefix = 0;  // high key bits decided so far
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      const uint32_t hi_mask = pass ? (0xFFFFFFFFu << (32 - 8 * pass)) : 0u;
      auto digit_of = [&](uint32_t u) { return int((u >> shift) & 0xFFu); };
      const int digit =
          short_list
              ? radix_pass(cand, ncand, hist, lane, want, at,
                           [&](uint32_t u) { return (u & hi_mask) == prefix; }, digit_of)
              : radix_pass(key, g.nbv, hist, lane, want, at,
                           [&](uint32_t u) { return (u & hi_mask) == prefix && in_bin(u); },
                           digit_of);
      prefix |= uint32_t(digit) << shift;
    }
    // prefix is now the exact key of the k-th best; `want` ties are needed
    const uint32_t thr = prefix;
    const int64_t row = int64_t(bh) * g.nb + g.nbp + i0 + warp;
    int32_t* out = idx + row * g.kcap;
    for (int p = lane; p < g.nbp; p += 32) out[p] = p;
    int written = g.nbp, ties = 0;
    if (want == at) {
      // every key equal to the k-th best is kept: take u >= thr
      for (int base = 0; base < g.nbv; base += 4 * 32) {
        uint32_t u[4];
        bool take[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int jv = base + 32 * i + lane;
          u[i] = jv < g.nbv ? key[jv] : 0u;
          take[i] = jv < g.nbv && u[i] >= thr;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t bal = __ballot_sync(0xffffffffu, take[i]);
          if (take[i]) out[written + __popc(bal & below)] = g.nbp + base + 32 * i + lane;
          written += __popc(bal);
        }
      }
    } else
    for (int base = 0; base < g.nbv; base += 4 * 32) {
      // four keys per lane loaded and voted on before the running counts
      uint32_t u[4], tie_bal[4];
      bool in[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int jv = base + 32 * i + lane;
        in[i] = jv < g.nbv;
        u[i] = in[i] ? key[jv] : 0u;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) tie_bal[i] = __ballot_sync(0xffffffffu, in[i] && u[i] == thr);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const bool tie = (tie_bal[i] >> lane) & 1u;
        const int tie_rank = ties + __popc(tie_bal[i] & below);
        const bool take = in[i] && (u[i] > thr || (tie && tie_rank < want));
        const uint32_t bal = __ballot_sync(0xffffffffu, take);
        if (take) out[written + __popc(bal & below)] = g.nbp + base + 32 * i + lane;
        written += __popc(bal);
        ties += __popc(tie_bal[i]);
      }
    }
    if (lane == 0) cnt[row] = g.nbp + g.keep;
  }
}

}  // namespace

cudaError_t launch_pool(const Geo& g, LayoutPtrs lp, const __nv_bfloat16* qp,
                        const __nv_bfloat16* kp, float* qpool, float* kpool, cudaStream_t st) {
  pool_kernel<<<dim3(g.nb, g.h, g.B), kPoolThreads, 0, st>>>(g, lp.bcount, qp, kp, qpool, kpool);
  return cudaGetLastError();
}

cudaError_t launch_pool_raster(const Geo& g, LayoutPtrs lp, const __nv_bfloat16* q,
                               const __nv_bfloat16* k, int64_t sb, int64_t sn, int64_t sh,
                               float* qpool, float* kpool, cudaStream_t st) {
  pool_raster_kernel<<<dim3(g.nb, g.h, g.B), kPoolThreads, 0, st>>>(g, lp.perm, lp.bcount, q, k,
                                                                    sb, sn, sh, qpool, kpool);
  return cudaGetLastError();
}

// shared memory of the untiled form (the limit a problem is validated against)
size_t select_smem_bytes(const Geo& g) {
  return sizeof(float) * kSelRows * g.d + sizeof(uint32_t) * kSelRows * g.nbv +
         sizeof(uint32_t) * (kSelThreads / 32) * 256;
}

namespace {
template <int KPT>
size_t select_tiled_smem_bytes(const Geo& g) {
  return sizeof(float) * kSelRows * g.d + sizeof(uint32_t) * ((kSelRows * g.nbv + 3) & ~3) +
         sizeof(float) * select_tile_floats<KPT>();
}

// the TMA form: the rows of RG groups, two 128-byte-swizzled chunk buffers
// (1024-byte aligned) and their two barriers
template <int KPT, int RG>
size_t select_tma_smem_bytes(const Geo& g) {
  const int rows = kSelRows * RG;
  return sizeof(float) * rows * g.d + sizeof(uint32_t) * ((rows * g.nbv + 3) & ~3) + 1024 +
         2 * size_t(kSelThreads) * KPT * kSelChunkTma * 4 + 16;
}

template <int KPT, bool TMA, int RG = 1>
cudaError_t launch_select_t(const Geo& g, size_t smem, const CUtensorMap* kmap,
                            const float* qpool, const float* kpool, const float* gate,
                            int32_t* idx, int32_t* cnt, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(select_kernel<KPT, TMA, RG>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  CUtensorMap none{};
  const int rows = kSelRows * RG;
  const int ctas = (g.nbv + rows - 1) / rows;
  select_kernel<KPT, TMA, RG><<<dim3(ctas, g.B * g.h), kSelThreads * RG, smem, st>>>(
      kmap ? *kmap : none, g, qpool, kpool, gate, idx, cnt);
  return cudaGetLastError();
}
}  // namespace

// The TMA-fed form when a pooled-key map is given and its buffers fit next
// to the row scores (16 query blocks per CTA, else 8); else the widest
// register tile that fits; else one key block per thread.
cudaError_t launch_select(const Geo& g, const float* qpool, const float* kpool, const float* gate,
                          const CUtensorMap* kmap, int32_t* idx, int32_t* cnt, cudaStream_t st) {
  constexpr size_t kMax = 227 * 1024;
  if (kmap && select_tma_smem_bytes<2, 2>(g) <= kMax)
    return launch_select_t<2, true, 2>(g, select_tma_smem_bytes<2, 2>(g), kmap, qpool, kpool,
                                       gate, idx, cnt, st);
  if (kmap && select_tma_smem_bytes<2, 1>(g) <= kMax)
    return launch_select_t<2, true>(g, select_tma_smem_bytes<2, 1>(g), kmap, qpool, kpool, gate,
                                    idx, cnt, st);
  if (select_tiled_smem_bytes<4>(g) <= kMax)
    return launch_select_t<4, false>(g, select_tiled_smem_bytes<4>(g), nullptr, qpool, kpool, gate,
                                     idx, cnt, st);
  if (select_tiled_smem_bytes<2>(g) <= kMax)
    return launch_select_t<2, false>(g, select_tiled_smem_bytes<2>(g), nullptr, qpool, kpool, gate,
                                     idx, cnt, st);
  if (select_tiled_smem_bytes<1>(g) <= kMax)
    return launch_select_t<1, false>(g, select_tiled_smem_bytes<1>(g), nullptr, qpool, kpool, gate,
                                     idx, cnt, st);
  return launch_select_t<0, false>(g, select_smem_bytes(g), nullptr, qpool, kpool, gate, idx, cnt,
                                   st);
}

}  // namespace bsa
