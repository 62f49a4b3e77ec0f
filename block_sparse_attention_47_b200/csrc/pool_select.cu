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
#include <cooperative_groups.h>

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
// The top-k of query rows i0 .. i0 + rows - 1 of (b, h) `bh` from their
// order keys (skey: [rows][nbv]), one warp per row: warp w takes row w with
// a 256-bin histogram at shist + 256 w and, when CAND > 0, a candidate list
// of CAND keys at scand + CAND w.  Writes the row's index list (prefix blocks
// first, then the kept video blocks ascending) and its count.
template <int CAND>
__device__ __forceinline__ void topk_rows(const Geo& g, const uint32_t* skey, uint32_t* shist,
                                          uint32_t* scand, int rows, int bh, int i0,
                                          int32_t* __restrict__ idx, int32_t* __restrict__ cnt,
                                          int warp, int lane) {
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
    uint32_t* cand = scand + warp * CAND;
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
  constexpr int CAND = KPT > 0 ? 512 : 0;
  topk_rows<CAND>(g, skey, shist, shist + ROWS * 256, rows, bh, i0, idx, cnt, warp, lane);
}


// ---- scores on the tensor cores, shared across a cluster --------------------
// A cluster of 8 CTAs takes 128 video query blocks of one (batch, head).  CTA
// c computes the scores of all 128 rows against its key blocks [c KC, (c+1)
// KC) on the tensor cores: tcgen05 kind::tf32, M = 128 rows, N = KC, K = 8
// channels per MMA, with every fp32 operand split as x = hi + lo (hi = x with
// its low 13 mantissa bits cleared, a tf32 value, so the split is exact) and
// S = qh.kh + qh.kl + ql.kh accumulated in fp32: the dropped ql.kl term and
// the tf32 truncation of each lo are each below 2^-20 |q||k| per channel,
// so a product is within 3 * 2^-20 |q||k| of the exact one.  Each CTA
// then stores every row's order keys into the shared memory of the CTA that
// owns the row (rows 16 c' .. 16 c' + 15 belong to CTA c'), and after a
// cluster barrier every CTA runs the same per-row top-k as the FMA kernels
// on its 16 rows.  One score tile of 128 x KC needs no global scratch: the
// 8 x 16 rows' keys live in the cluster's shared memory.
constexpr int kTcCluster = 8, kTcM = 128, kTcRows = kTcM / kTcCluster;
constexpr int kTcThreads = 512;
constexpr int kTcMaxKeys = kTcCluster * 256;  // N <= 256 per CTA
constexpr uint32_t kTcCols = 256;
// shared memory from the 1024-byte-aligned base: query hi/lo tiles per
// 32-channel chunk (32 KB each), then the query rows in fp32 and later the
// key hi/lo stage (64 KB), then the barrier; after the scores the first
// 176 KB hold the row keys [16][nbv], histograms [16][256] and candidate
// lists [16][512]
constexpr uint32_t kTcChunk = 32768, kTcOffBar = 196608;
constexpr uint32_t kTcOffHist = 131072, kTcOffCand = kTcOffHist + 16384;
constexpr size_t kTcSmem = kTcOffBar + 64 + 1024;
static_assert(kTcOffCand + 4 * kTcRows * 512 <= kTcOffBar, "top-k space");
static_assert(4 * kTcRows * kTcMaxKeys <= kTcOffHist, "row keys");

// instruction descriptor of kind::tf32: fp32 accumulator (bits 4-5 = 1),
// A and B tf32 (format 2 in bits 7-9 and 10-12), both K-major
__host__ __device__ constexpr uint32_t idesc_tf32_f32(int M, int N) {
  return (1u << 4) | (2u << 7) | (2u << 10) | (uint32_t(N >> 3) << 17) |
         (uint32_t(M >> 4) << 24);
}

__device__ __forceinline__ void tc_mma_tf32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

// x with the low 13 mantissa bits cleared: exactly representable in tf32
__device__ __forceinline__ float tf32_hi(float x) {
  return __uint_as_float(__float_as_uint(x) & 0xFFFFE000u);
}

// hi and lo parts of four channels into 16-byte unit u of row r of two
// 128-byte-swizzled operand tiles
__device__ __forceinline__ void store_split(uint32_t hi_tile, uint32_t lo_tile, int r, int u,
                                            float4 x) {
  const float4 h = make_float4(tf32_hi(x.x), tf32_hi(x.y), tf32_hi(x.z), tf32_hi(x.w));
  const float4 l = make_float4(x.x - h.x, x.y - h.y, x.z - h.z, x.w - h.w);
  const uint32_t off = uint32_t(r) * 128u + ((uint32_t(u) ^ uint32_t(r & 7)) << 4);
  st_shared_v4(hi_tile + off, make_uint4(__float_as_uint(h.x), __float_as_uint(h.y),
                                         __float_as_uint(h.z), __float_as_uint(h.w)));
  st_shared_v4(lo_tile + off, make_uint4(__float_as_uint(l.x), __float_as_uint(l.y),
                                         __float_as_uint(l.z), __float_as_uint(l.w)));
}

__global__ void __cluster_dims__(kTcCluster, 1, 1) __launch_bounds__(kTcThreads, 1)
    select_tc_kernel(Geo g, int KC, const float* __restrict__ qpool,
                     const float* __restrict__ kpool, const float* __restrict__ gate,
                     int32_t* __restrict__ idx, int32_t* __restrict__ cnt,
                     int32_t* __restrict__ status) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* sm = smem_raw + (base - raw);
  const int nch = g.d / 32;                    // 32-channel chunks
  const uint32_t sA = base, sR = base + uint32_t(nch) * kTcChunk;
  float* sq = reinterpret_cast<float*>(sm + uint32_t(nch) * kTcChunk);
  const uint32_t bar = base + kTcOffBar;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + kTcOffBar + 8);
  uint32_t* skey = reinterpret_cast<uint32_t*>(sm);
  uint32_t* shist = reinterpret_cast<uint32_t*>(sm + kTcOffHist);
  uint32_t* scand = reinterpret_cast<uint32_t*>(sm + kTcOffCand);

  const int crank = int(cluster.block_rank());
  const int bh = blockIdx.y, r0 = (blockIdx.x / kTcCluster) * kTcM;  // first query block
  const int k0 = crank * KC, nk = min(KC, g.nbv - k0);               // this CTA's keys
  const int64_t pool0 = int64_t(bh) * g.nb * g.d;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // prefix query blocks attend densely: mark them once per (b, h)
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < g.nbp; i += kTcThreads) cnt[int64_t(bh) * g.nb + i] = -1;
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_holder), kTcCols);
    tmem_relinquish();
  }
  for (int e = threadIdx.x; e < kTcM * g.d / 4; e += kTcThreads) {
    const int r = e / (g.d / 4), c4 = e % (g.d / 4);
    reinterpret_cast<float4*>(sq)[e] =
        r0 + r < g.nbv ? __ldg(reinterpret_cast<const float4*>(
                             qpool + pool0 + int64_t(g.nbp + r0 + r) * g.d) + c4)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  if (gate) {
    // q~ = G q: this CTA maps the 16 rows it owns (the FMA kernels' fmaf
    // chains) and stores them into every CTA's copy of the rows, once every
    // CTA has loaded its plain rows
    cluster.sync();
    const float* G = gate + int64_t(bh % g.h) * g.d * g.d;
    constexpr int MAXO = kTcRows * 128 / kTcThreads;
    const int c = threadIdx.x % g.d, q0 = threadIdx.x / g.d, qstep = kTcThreads / g.d;
    const int nout = kTcRows * g.d / kTcThreads;
    const int mine = crank * kTcRows;
    float acc[MAXO];
#pragma unroll
    for (int o = 0; o < MAXO; ++o) acc[o] = 0.f;
    const float4* gr = reinterpret_cast<const float4*>(G + int64_t(c) * g.d);
    // eight loads of the gate row in flight (d / 4 is a multiple of 8)
#pragma unroll 8
    for (int e4 = 0; e4 < g.d / 4; ++e4) {
      const float4 gv = __ldg(gr + e4);
#pragma unroll
      for (int o = 0; o < MAXO; ++o) {
        if (o < nout) {
          const float4 qv =
              reinterpret_cast<const float4*>(sq + (mine + q0 + qstep * o) * g.d)[e4];
          acc[o] = fmaf(gv.x, qv.x, acc[o]);
          acc[o] = fmaf(gv.y, qv.y, acc[o]);
          acc[o] = fmaf(gv.z, qv.z, acc[o]);
          acc[o] = fmaf(gv.w, qv.w, acc[o]);
        }
      }
    }
    __syncthreads();  // this CTA's own rows are read before they are replaced
#pragma unroll 1
    for (int dst = 0; dst < kTcCluster; ++dst) {
      float* rq = cluster.map_shared_rank(sq, dst);
#pragma unroll
      for (int o = 0; o < MAXO; ++o)
        if (o < nout) rq[(mine + q0 + qstep * o) * g.d + c] = acc[o];
    }
    cluster.sync();  // every CTA's rows are mapped
  }
  // the query rows as A tiles: [chunk][128 rows][32 channels], hi and lo
  for (int e = threadIdx.x; e < kTcM * g.d / 4; e += kTcThreads) {
    const int r = e / (g.d / 4), c4 = e % (g.d / 4);
    store_split(sA + (c4 / 8) * kTcChunk, sA + (c4 / 8) * kTcChunk + 16384, r, c4 % 8,
                reinterpret_cast<const float4*>(sq)[e]);
  }
  __syncthreads();  // sq is dead: its space takes the key stage
  // key chunks: [ntk x 128 rows][32 channels], hi at sR, lo at sR + 32 KB;
  // a chunk's global loads are issued before the previous chunk's MMAs are
  // waited for.  The keys are the MMA's A (M = 128 per key tile), the query
  // rows its B (N = 128), so that tensor-memory lane = key and a warp's
  // stores of one row's scores are contiguous.
  const int ntk = (KC + 127) / 128;
  const int units = ntk * 128 * 8;  // 16-byte units of a chunk
  constexpr int UPT = 2 * 128 * 8 / kTcThreads;
  float4 x[UPT];
  auto fetch = [&](int cc) {
#pragma unroll
    for (int i = 0; i < UPT; ++i) {
      const int e = threadIdx.x + i * kTcThreads;
      const int kr = e >> 3, u = e & 7;
      x[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (e < units && kr < nk)
        x[i] = __ldg(reinterpret_cast<const float4*>(kpool + pool0 +
                                                     int64_t(g.nbp + k0 + kr) * g.d + cc * 32) +
                     u);
    }
  };
  constexpr uint32_t idesc = idesc_tf32_f32(128, kTcM);
  bool ok = true;
  fetch(0);
  for (int cc = 0; cc < nch; ++cc) {
    // the stage was last read by chunk cc - 1's MMAs
    if (cc > 0) ok = mbar_wait(bar, (cc - 1) & 1, nullptr) && ok;
#pragma unroll
    for (int i = 0; i < UPT; ++i) {
      const int e = threadIdx.x + i * kTcThreads;
      if (e < units) store_split(sR, sR + 32768, e >> 3, e & 7, x[i]);
    }
    if (cc + 1 < nch) fetch(cc + 1);
    fence_proxy_async_smem();
    __syncthreads();
    if (threadIdx.x == 0) {
      tc_fence_after();
      const uint32_t qh0 = sA + cc * kTcChunk, ql0 = qh0 + 16384;
      for (int t = 0; t < ntk; ++t) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {  // 8 channels (32 bytes) per MMA
          const uint64_t ah = sdesc_sw128(sR + t * 16384 + k * 32, 16, 1024);
          const uint64_t al = sdesc_sw128(sR + 32768 + t * 16384 + k * 32, 16, 1024);
          const uint64_t bq = sdesc_sw128(qh0 + k * 32, 16, 1024);
          const uint64_t bl = sdesc_sw128(ql0 + k * 32, 16, 1024);
          const uint32_t d_t = tmem + 128u * uint32_t(t);
          tc_mma_tf32(d_t, ah, bq, idesc, (cc > 0 || k > 0) ? 1u : 0u);
          tc_mma_tf32(d_t, ah, bl, idesc, 1u);
          tc_mma_tf32(d_t, al, bq, idesc, 1u);
        }
      }
      tc_commit(bar);
    }
  }
  ok = mbar_wait(bar, (nch - 1) & 1, nullptr) && ok;
  if (!ok && threadIdx.x == 0) atomicCAS(status, 0, int32_t(BSA_ERR_TIMEOUT));
  tc_fence_after();
  // every CTA's MMAs are done with its staging space, which now takes the
  // row keys that the other CTAs store into it
  cluster.sync();
  {
    // warp w reads TMEM lanes 32 (w % 4) .. (keys) of key tile t = w / 8,
    // columns (query rows) 64 ((w / 4) % 2) .. + 63, 16 at a time: rows
    // 16 c' .. 16 c' + 15 go to CTA c', from key k0 on
    const int quarter = warp & 3, t = warp >> 3, rh = (warp >> 2) & 1;
    const int kl = 128 * t + 32 * quarter + lane;  // this lane's key, from k0
    if (t < ntk) {
#pragma unroll 1
      for (int cb = 0; cb < 4; ++cb) {
        uint32_t v[16];
        tmem_ld16(tmem + (uint32_t(quarter * 32) << 16) + 128u * uint32_t(t) +
                      uint32_t(64 * rh + 16 * cb),
                  v);
        uint32_t* dst = cluster.map_shared_rank(skey, 4 * rh + cb) + k0 + kl;
        if (kl < nk)
#pragma unroll
          for (int i = 0; i < 16; ++i) dst[i * g.nbv] = order_key(__uint_as_float(v[i]));
      }
    }
  }
  tc_fence_before();
  cluster.sync();  // every row's keys have arrived
  const int i0 = r0 + crank * kTcRows;
  const int rows = max(0, min(kTcRows, g.nbv - i0));
  topk_rows<512>(g, skey, shist, scand, rows, bh, i0, idx, cnt, warp, lane);
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTcCols);
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
                          const CUtensorMap* kmap, int32_t* idx, int32_t* cnt, int32_t* status,
                          cudaStream_t st) {
  constexpr size_t kMax = 227 * 1024;
  if (g.nbv <= kTcMaxKeys && (g.d == 64 || g.d == 128)) {
    // the tensor-core form: 8-CTA clusters of 128 query blocks, KC keys per
    // CTA (a multiple of 16, the MMA's N)
    const int KC = ((g.nbv + 16 * kTcCluster - 1) / (16 * kTcCluster)) * 16;
    cudaError_t e = cudaFuncSetAttribute(select_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(kTcSmem));
    if (e != cudaSuccess) return e;
    const int tiles = (g.nbv + kTcM - 1) / kTcM;
    select_tc_kernel<<<dim3(tiles * kTcCluster, g.B * g.h), kTcThreads, kTcSmem, st>>>(
        g, KC, qpool, kpool, gate, idx, cnt, status);
    return cudaGetLastError();
  }
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
