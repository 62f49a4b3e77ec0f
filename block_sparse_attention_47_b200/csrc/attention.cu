// Block-sparse attention forward on sm_100a: TMA-fed tcgen05 tiles with the
// accumulators and the A operands in tensor memory, walking a per-query-block
// list of kept key blocks so that only kept 64x64 tiles are ever loaded or
// multiplied (Sparse VideoGen on TPU, aibase.it, section "이론적 sparsity와
// 물리적 sparsity의 차이": skipping empty tiles is where the speed comes
// from).
//
// CTA = two adjacent query blocks (128 query rows = the full tcgen05 M=128
// datapath; M=64 would leave half of it idle).  The union of the two
// blocks' key lists is the CTA's sequence of steps, one 64-token key block
// each.  Steps go in pairs (one per softmax warpgroup) and each pair's
// scores come from one full-width MMA burst:
//     [S_j | S_j+1] = Q [K_j ; K_j+1]^T   M=128, N=128, K=head_dim
//     O_w += P_j V_j                      M=128, N=head_dim, K=64
// with A = Q or P read from TMEM and B = K or V from shared memory.  Every
// MMA burst pays a pipeline-fill latency, so fewer, wider bursts keep the
// tensor pipe busier.  Rows of a block that did not keep the step's key
// block get P = 0.
//
// K and V sit in separate shared-memory rings: a K stage is recycled as
// soon as its score burst has run, a V stage after its PV, so K is fetched
// several steps ahead of its use and the TMA latency (far L2 partition or
// HBM) stays hidden.  The K ring is box-major so that the K blocks of two
// consecutive stages are contiguous (one B operand for the pair burst).
// Ring discipline: every wait on a ring barrier must be at most one phase
// away from the phase it tests (a parity wait cannot tell phases two apart).
// The K ring has an even number of stages, so a stage is reused only by
// steps of one parity and each K copy warp serves one parity in order.  A V
// stage is reused by both parities (odd ring), so each V copy warp copies
// one 64-column box of every step in order, and PVs are issued in step
// order.
//
// Two softmax warpgroups take alternate steps, each with its own running
// max, running sum and O accumulator (an exact split of the key set); the
// epilogue merges them: O = (a0*O0 + a1*O1) / (a0*l0 + a1*l1),
// a_w = 2^(m_w - max(m0, m1)).  The softmax is the exact online softmax in
// the exp2 domain with a lazily updated running max: O is rescaled only
// when the row max grows by more than 8 (so every probability stays below
// 2^8), which is still exact after the final division.
//
// The step sequence is fixed before the walk starts: warp 8 turns the two
// index lists into bitmaps over the key blocks (one bit per kept block) and
// expands their union A|B into a table of 16-bit step entries in shared
// memory (key block and flags), 32-block words in a rotated order and bits
// ascending within a word.  Every role reads step j straight from the table,
// so no role waits for another to hand it the next key block.
//
// Warp roles (512 threads):
//   warps 0-3 / 4-7  softmax warpgroup 0 / 1; thread r of a group owns
//                    query row r = TMEM lane r (warp w reaches lanes
//                    32*(w%4)..+31); group 0 first copies Q into TMEM
//   warp 8           builds the step bitmaps, then copies box 0 (head_dim
//                    0-63) of even steps' K
//   warp 9           TMEM allocator; one thread issues the score bursts
//   warp 10          K box 0 of odd steps
//   warps 11 / 12    K box 1 (head_dim 64-127) of even / odd steps
//   warp 13          one thread issues the PV MMAs of both softmax groups
//   warps 14 / 15    V box 0 / box 1 of every step
// One issuing thread completes about one bulk tensor copy per ~650 cycles
// whatever its size, so copies are spread over six warps; tcgen05.mma
// blocks its issuing thread while the tensor pipe is busy, so score bursts
// and PVs come from two threads.
// Tensor memory (512 columns): Q [0,64) bf16 pairs | S0 [64,128) | S1
// [128,192) | P0 [192,224) | P1 [224,256) | O0 [256,384) | O1 [384,512).
//
// Every wait is bounded (2 s); a timeout sets the caller's status word to
// BSA_ERR_TIMEOUT, drains in-flight copies and MMAs and frees tensor memory.
#include "bsa_internal.cuh"

namespace bsa {
namespace {

constexpr int kMaxWords = kAttnMaxBlocks / 32;  // step-bitmap words per query block
// step table entry: key block in bits 0-12, then the first query block keeps
// it (bit 13), the second one does (bit 14), all 64 slots are real tokens (15)
constexpr uint32_t kTileMask = 0x1FFFu, kFlagShift = 13;
static_assert(kAttnMaxBlocks <= 8192, "13-bit key block in a step entry");

template <int D>
struct Cfg {
  static constexpr int kThreads = 512;
  static constexpr int KB = D / 64;  // 64-column boxes per block (copy streams per ring)
  static constexpr int KS = 8;                    // K ring stages (even: pairs)
  static constexpr int VS = 5;                    // V ring stages
  static constexpr int BLK_BYTES = 64 * D * 2;    // one K (or V) block
  static constexpr int BOX = 64 * 128;            // one 64-column TMA box of a block
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_Q = 0, COL_S = 64, COL_P = 192, COL_O = 256;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = KS * BLK_BYTES;
  static constexpr int OFF_BAR = OFF_V + VS * BLK_BYTES;
  // kfull[KS] kempty[KS] vfull[VS] vempty[VS] qready s sfree[2] p[2] o[2] drain[2] steps
  static constexpr int N_BARS = 2 * KS + 2 * VS + 12;
  static constexpr int OFF_XCH = OFF_BAR + 8 * N_BARS;  // float m[2][128], l[2][128]
  static constexpr int OFF_BM = OFF_XCH + 4 * 4 * 128;   // uint32 A, B, F [kMaxWords]
  static constexpr int OFF_STEPS = OFF_BM + 3 * 4 * kMaxWords;  // uint16 [kAttnMaxBlocks]
  static constexpr int OFF_MISC = OFF_STEPS + 2 * kAttnMaxBlocks;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;  // + slack for 1024-B alignment
  static_assert(KS % 2 == 0, "step pairs must not straddle the K ring's end");
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

__device__ __forceinline__ void report_timeout(volatile int* abort_flag, int32_t* status) {
  *abort_flag = 1;
  atomicCAS(status, 0, int32_t(BSA_ERR_TIMEOUT));
}

// Non-blocking probe of an mbarrier phase that is only issued once `dep`
// has been computed: it lands among the exponentials, and its ~150-cycle
// latency is spent on the ones that follow it.
__device__ __forceinline__ bool mbar_test_after(uint32_t bar, uint32_t parity, float dep) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "f"(dep)
      : "memory");
  return ok != 0;
}

// 2^x for two lanes on the FMA pipe, for a share of the exponentials so that
// the MUFU unit is not the only one working: 2^x = 2^n * 2^f with n the
// nearest integer (from adding 1.5 * 2^23) and f in [-0.5, 0.5]; 2^f by a
// degree-3 least-squares fit on Chebyshev nodes (relative error below
// 7.8e-5, well under the bf16 rounding of P), and n added to the exponent
// field.  x is clamped at -125 so that the result stays a normal number.
__device__ __forceinline__ void exp2_poly_x2(float& y0, float& y1, float x0, float x1) {
  constexpr float kRound = 12582912.f;  // 1.5 * 2^23
  constexpr float c0 = 0.99992895f, c1 = 0.69327623f, c2 = 0.24260405f, c3 = 0.05508868f;
  x0 = fmaxf(x0, -125.f);
  x1 = fmaxf(x1, -125.f);
  float t0, t1, n0, n1, f0, f1, p0, p1;
  add_f32x2(t0, t1, x0, x1, kRound, kRound);
  add_f32x2(n0, n1, t0, t1, -kRound, -kRound);
  add_f32x2(f0, f1, x0, x1, -n0, -n1);
  fma_f32x2(p0, p1, f0, f1, c3, c3, c2, c2);
  fma_f32x2(p0, p1, p0, p1, f0, f1, c1, c1);
  fma_f32x2(p0, p1, p0, p1, f0, f1, c0, c0);
  // the low bits of t hold n (two's complement); shifted into the exponent
  // field, the constant's own bits fall off the top
  y0 = __int_as_float(__float_as_int(p0) + int(uint32_t(__float_as_int(t0)) << 23));
  y1 = __int_as_float(__float_as_int(p1) + int(uint32_t(__float_as_int(t1)) << 23));
}

__device__ __forceinline__ bool bit_of(uint32_t lo, uint32_t hi, int c) {
  return ((c < 32 ? (lo >> c) : (hi >> (c - 32))) & 1u) != 0u;
}

// The box of video block t (t >= nbp) of batch element b: origin
// (t0, y0, x0) on the grid and sides (st, sh, sw); returns its shape code
// (0 = 4x4x4).  Its 64 slots hold the box's tokens in (t, y, x) order.
struct Box {
  int t0, y0, x0, st, sh, sw;
};

__device__ __forceinline__ int video_block_box(const Geo& g, const uint8_t* __restrict__ codes,
                                               int b, int t, Box& bx) {
  const int jv = t - g.nbp;
  if (g.mode == BSA_BLOCK_FIXED_444) {
    const int nbh = g.H >> 2, nbw = g.W >> 2;
    const int bt = jv / (nbh * nbw), rem = jv - bt * (nbh * nbw);
    const int bhh = rem / nbw;
    bx = {4 * bt, 4 * bhh, 4 * (rem - bhh * nbw), 4, 4, 4};
    return 0;
  }
  const int r = jv >> 3, sub = jv & 7;
  const int nrh = g.H >> 3, nrw = g.W >> 3;
  const int rt = r / (nrh * nrw), rem = r - rt * (nrh * nrw);
  const int rh = rem / nrw, rw = rem - rh * nrw;
  int code = __ldg(codes + int64_t(b) * g.nreg + r);
  code = code > 6 ? 0 : code;
  int st, sh, sw;
  shape_sides(code, st, sh, sw);
  const int gh = 8 / sh, gw = 8 / sw;
  const int bt = sub / (gh * gw), bhh = (sub / gw) % gh, bw = sub % gw;
  bx = {8 * rt + st * bt, 8 * rh + sh * bhh, 8 * rw + sw * bw, st, sh, sw};
  return code;
}

// One K (or V) copy: box bx (64 head_dim columns) of key block t of
// (batch, head) bh into shared memory at dst.  Block order: one 3-D box of
// the permuted tensor.  Raster order: a prefix block is 64 consecutive
// tokens (3-D map over [B, N, heads*d]); a video block is one 5-D box
// {64 columns, sw, sh, st, 1} of the [B, T, H, W, heads*d] grid whose rows
// land in shared memory in (t, y, x) order, i.e. in slot order, so the
// shared-memory tile is the same as the permuted one.
template <int D, bool RASTER>
__device__ __forceinline__ void kv_copy(uint32_t dst, const KVMaps<RASTER>& maps, bool is_k,
                                        uint32_t bar, int bx, int t, int bh, const Geo& g,
                                        const uint8_t* __restrict__ codes) {
  if constexpr (!RASTER) {
    tma_load_3d(dst, is_k ? &maps.k : &maps.v, bar, 64 * bx, t * 64, bh);
  } else {
    const int b = bh / g.h, c0 = (bh - b * g.h) * D + 64 * bx;
    const CUtensorMap* m = is_k ? maps.k : maps.v;
    if (t < g.nbp) {
      tma_load_3d(dst, m, bar, c0, t * 64, b);
      return;
    }
    Box box;
    const int code = video_block_box(g, codes, b, t, box);
    tma_load_5d(dst, m + 1 + code, bar, c0, box.x0, box.y0, box.t0, b);
  }
}

// ---- window heads ------------------------------------------------------------
// A window head (Sparse VideoGen on TPU, aibase.it, section "Sparse
// VideoGen의 핵심 아이디어": spatial heads look within nearby frames,
// temporal heads at the same place across frames) lets query token
// (t, y, x) see video key (t', y', x') when |t' - t| <= w_t, |y' - y| <= w_y
// and |x' - x| <= w_x, a negative w leaving that axis free; prefix keys and
// prefix queries stay dense.  A tile is empty when, on some axis, the two
// blocks' extents are farther apart than the window (skipped: not in the
// walk), full when every pair is inside, boundary otherwise (an element mask
// per query row, built from the key block's box).

// 1 when some pair of the extents [a0, a0+la) and [b0, b0+lb) is within w
__device__ __forceinline__ bool axis_reach(int a0, int la, int b0, int lb, int w) {
  if (w < 0) return true;
  const int gap = max(0, max(b0 - (a0 + la - 1), a0 - (b0 + lb - 1)));
  return gap <= w;
}

// bits [lo, hi) of a 64-bit word (0 when lo >= hi)
__device__ __forceinline__ uint64_t bit_range(int lo, int hi) {
  lo = max(lo, 0);
  hi = min(hi, 64);
  if (lo >= hi) return 0ull;
  const uint64_t up = hi >= 64 ? ~0ull : ((1ull << hi) - 1ull);
  return up & ~((1ull << lo) - 1ull);
}

// slots s of a key block whose coordinate along one axis, k0 + (s / inner)
// % side, lies in [q - w, q + w]: a run of `inner`-wide groups repeated with
// period inner*side (a divisor of 64)
__device__ __forceinline__ uint64_t axis_bits(int q, int w, int k0, int side, int inner) {
  if (w < 0) return ~0ull;
  const int lo = max(q - w - k0, 0), hi = min(q + w - k0, side - 1);
  if (lo > hi) return 0ull;
  const int period = inner * side;
  const uint64_t one = bit_range(lo * inner, (hi + 1) * inner);
  const uint64_t comb = period >= 64 ? 1ull : (~0ull / ((1ull << period) - 1ull));
  return one * comb;
}

// element mask of one query row (video token at tq, yq, xq) for a video key block
__device__ __forceinline__ uint64_t window_bits(const Box& k, int tq, int yq, int xq, int wt,
                                                int wy, int wx) {
  return axis_bits(tq, wt, k.t0, k.st, k.sh * k.sw) & axis_bits(yq, wy, k.y0, k.sh, k.sw) &
         axis_bits(xq, wx, k.x0, k.sw, 1);
}

// what decides a CTA's walk: index lists, every block, or per-head windows
enum { kModeLists = 0, kModeDense = 1, kModeWindow = 2 };

template <int D, int MODE, bool RASTER>
__global__ void __launch_bounds__(512, 1)
    attn_fwd_kernel(const __grid_constant__ KVMaps<RASTER> maps, Geo g, const AttnIO io) {
  using C = Cfg<D>;
  const uint64_t* __restrict__ bmask = io.bmask;
  const uint8_t* __restrict__ bfull = io.bfull;
  const int32_t* __restrict__ idx = io.idx;
  const int32_t* __restrict__ cnt = io.cnt;
  int32_t* __restrict__ status = io.status;
  constexpr int KS = C::KS, VS = C::VS;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* sm = smem_raw + (base - raw);
  const uint32_t sK = base + C::OFF_K, sV = base + C::OFF_V, bar0 = base + C::OFF_BAR;
  auto kfull = [&](int s) { return bar0 + 8u * uint32_t(s); };
  auto kempty = [&](int s) { return bar0 + 8u * uint32_t(KS + s); };
  auto vfull = [&](int s) { return bar0 + 8u * uint32_t(2 * KS + s); };
  auto vempty = [&](int s) { return bar0 + 8u * uint32_t(2 * KS + VS + s); };
  auto ful_of = [&](bool k, int s) { return k ? kfull(s) : vfull(s); };
  const uint32_t bar_qready = bar0 + 8u * (2 * KS + 2 * VS);
  const uint32_t bar_s = bar_qready + 8;       // S of a step pair ready
  const uint32_t bar_sfree = bar_qready + 16;  // both groups have read their S (256 arrivals)
  const uint32_t bar_p = bar_qready + 32;      // [2] P written + O corrected (128 arrivals)
  const uint32_t bar_o = bar_qready + 48;      // [2] PV of group w finished
  const uint32_t bar_drain = bar_qready + 64;  // [2] score issuer, PV issuer
  const uint32_t bar_steps = bar_qready + 80;  // step bitmaps built (32 arrivals)
  uint32_t* bmA = reinterpret_cast<uint32_t*>(sm + C::OFF_BM);  // first query block's keys
  uint32_t* bmB = bmA + kMaxWords;                                 // second query block's keys
  uint32_t* bmF = bmA + 2 * kMaxWords;                             // key blocks with no pad slot
  uint16_t* steps = reinterpret_cast<uint16_t*>(sm + C::OFF_STEPS);  // the walk, in order
  float* xch = reinterpret_cast<float*>(sm + C::OFF_XCH);  // m[2][128] then l[2][128]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + C::OFF_MISC + 4);
  int* n_steps_sm = reinterpret_cast<int*>(sm + C::OFF_MISC + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x, bh = blockIdx.y, b = bh / g.h;

  // the step-table warp issues all of its global loads before the set-up
  // barrier, so that their latencies overlap it and one another: the two
  // lists' lengths, their first 256 entries (read up to the lists' capacity,
  // since the lengths are not known yet) and the full-block flags of the
  // first 64 bitmap words
  int pre_cnt[2] = {-1, -1};
  int pre_a[8], pre_b[8];
  uint32_t pre_f[2][8];
  if (warp == 8) {
    if constexpr (MODE == kModeLists) {
      const int32_t* srcA = idx + (int64_t(bh) * g.nb + 2 * pair) * g.kcap;
      const bool has_b = 2 * pair + 1 < g.nb;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf)
        if (2 * pair + hf < g.nb) pre_cnt[hf] = __ldg(cnt + int64_t(bh) * g.nb + 2 * pair + hf);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = 32 * u + lane;
        pre_a[u] = i < g.kcap ? __ldg(srcA + i) : -1;
        pre_b[u] = i < g.kcap && has_b ? __ldg(srcA + g.kcap + i) : -1;
      }
    }
    const uint32_t* f4 = reinterpret_cast<const uint32_t*>(bfull + int64_t(b) * g.nb);
    const bool words = ((int64_t(b) * g.nb) & 3) == 0;  // 4-byte aligned flags
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int w = lane + 32 * r;
#pragma unroll
      for (int i = 0; i < 8; ++i)
        pre_f[r][i] = words && 32 * w + 32 <= g.nb ? __ldg(f4 + 8 * w + i) : 0u;
    }
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < KS; ++s) {
      mbar_init(kfull(s), C::KB);
      mbar_init(kempty(s), 1);
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(vfull(s), C::KB);
      mbar_init(vempty(s), 1);
    }
    mbar_init(bar_qready, 128);
    mbar_init(bar_s, 1);
    mbar_init(bar_sfree, 256);
    for (int w = 0; w < 2; ++w) {
      mbar_init(bar_p + 8 * w, 128);
      mbar_init(bar_o + 8 * w, 1);
    }
    mbar_init(bar_drain, 1);
    mbar_init(bar_drain + 8, 1);
    mbar_init(bar_steps, 32);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int nw = (g.nb + 31) >> 5;
  const int ws = int((uint32_t(pair) * 61u + uint32_t(bh) * 17u) % uint32_t(nw));

  if (warp == 8 || warp == 10 || warp == 11 || warp == 12 || warp == 14 || warp == 15) {
    if (warp == 8) {
      // ------------------------------------------------------ step bitmaps
      // Bit t of A (B) is set when the first (second) query block of the
      // pair keeps key block t; a dense row keeps every block.  Entries
      // outside 0..nb-1 are ignored rather than trusted.
      for (int w = lane; w < nw; w += 32) {
        bmA[w] = 0u;
        bmB[w] = 0u;
      }
      __syncwarp();
      for (int hf = 0; hf < 2; ++hf) {
        const int qb = 2 * pair + hf;
        if (qb >= g.nb) continue;
        uint32_t* bm = hf ? bmB : bmA;
        if constexpr (MODE == kModeWindow) {
          // a video query block walks the prefix and every video key block
          // its box can reach through the window (non-empty tiles)
          if (qb >= g.nbp) {
            const int32_t* win = io.windows + 3 * (bh - b * g.h);
            const int wt = __ldg(win), wy = __ldg(win + 1), wx = __ldg(win + 2);
            Box qx;
            video_block_box(g, io.codes, b, qb, qx);
            for (int w = 0; w < nw; ++w) {
              const int j = 32 * w + lane;
              bool on = j < g.nbp;
              if (j >= g.nbp && j < g.nb) {
                Box kx;
                video_block_box(g, io.codes, b, j, kx);
                on = axis_reach(qx.t0, qx.st, kx.t0, kx.st, wt) &&
                     axis_reach(qx.y0, qx.sh, kx.y0, kx.sh, wy) &&
                     axis_reach(qx.x0, qx.sw, kx.x0, kx.sw, wx);
              }
              const uint32_t word = __ballot_sync(0xffffffffu, on);
              if (lane == 0) bm[w] = word;
            }
            continue;
          }
        }
        // a dense row keeps every block (lists are read below, both at once)
        if (MODE != kModeLists || pre_cnt[hf] < 0) {
          for (int w = lane; w < nw; w += 32) {
            const int rem = g.nb - 32 * w;
            bm[w] = rem >= 32 ? ~0u : ((1u << rem) - 1u);
          }
        }
      }
      if constexpr (MODE == kModeLists) {
        // the two index lists, loaded together so that their latencies overlap
        const int nA = pre_cnt[0] < 0 ? 0 : (pre_cnt[0] < g.kcap ? pre_cnt[0] : g.kcap);
        const int nB = pre_cnt[1] < 0 ? 0 : (pre_cnt[1] < g.kcap ? pre_cnt[1] : g.kcap);
        const int32_t* srcA = idx + (int64_t(bh) * g.nb + 2 * pair) * g.kcap;
        const int32_t* srcB = srcA + g.kcap;
        const int nmax = nA > nB ? nA : nB;
        for (int base = 0; base < nmax; base += 8 * 32) {
          int va[8], vb[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int i = base + 32 * u + lane;
            // the first 256 entries were loaded before the set-up barrier
            va[u] = i >= nA ? -1 : (base == 0 ? pre_a[u] : __ldg(srcA + i));
            vb[u] = i >= nB ? -1 : (base == 0 ? pre_b[u] : __ldg(srcB + i));
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            if (va[u] >= 0 && va[u] < g.nb) atomicOr(bmA + (va[u] >> 5), 1u << (va[u] & 31));
            if (vb[u] >= 0 && vb[u] < g.nb) atomicOr(bmB + (vb[u] >> 5), 1u << (vb[u] & 31));
          }
        }
      }
      // F: blocks whose 64 slots are all real tokens (no valid-slot mask needed)
      const uint8_t* full_row = bfull + int64_t(b) * g.nb;
      const bool words = ((int64_t(b) * g.nb) & 3) == 0;  // 4-byte aligned flags
      for (int w = lane; w < nw; w += 32) {
        uint32_t f = 0u;
        if (words && 32 * w + 32 <= g.nb) {
          // eight 4-byte words of the 32 flag bytes (each byte 0 or 1); those
          // of the first 64 bitmap words were loaded before the set-up barrier
          const uint32_t* f4 = reinterpret_cast<const uint32_t*>(full_row + 32 * w);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint32_t x = w < 32 ? pre_f[0][i] : (w < 64 ? pre_f[1][i] : __ldg(f4 + i));
            f |= (((x & 0xFFu) != 0u) | (((x >> 8) & 0xFFu) != 0u) << 1 |
                  (((x >> 16) & 0xFFu) != 0u) << 2 | ((x >> 24) != 0u) << 3) << (4 * i);
          }
        } else {
          for (int i = 0; i < 32; ++i)
            if (32 * w + i < g.nb && __ldg(full_row + 32 * w + i)) f |= 1u << i;
        }
        bmF[w] = f;
      }
      __syncwarp();
      // the step table: set bits of A|B, words in the rotated order ws, ws+1,
      // .., nw-1, 0, .., ws-1 and bits ascending within a word; lane l takes
      // word l of each round of 32 and writes at its prefix-sum offset
      int nsteps = 0;
      for (int r0 = 0; r0 < nw; r0 += 32) {
        const int pos = r0 + lane;
        const int w = pos < nw ? (ws + pos < nw ? ws + pos : ws + pos - nw) : 0;
        const uint32_t a = pos < nw ? bmA[w] : 0u, bb = pos < nw ? bmB[w] : 0u;
        const uint32_t f = pos < nw ? bmF[w] : 0u;
        uint32_t u = a | bb;
        const int c = __popc(u);
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        int at = nsteps + incl - c;
        while (u) {
          const int bit = __ffs(u) - 1;
          u &= u - 1u;
          steps[at++] = uint16_t(uint32_t(32 * w + bit) | (((a >> bit) & 1u) << kFlagShift) |
                                 (((bb >> bit) & 1u) << (kFlagShift + 1)) |
                                 (((f >> bit) & 1u) << (kFlagShift + 2)));
        }
        nsteps += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (lane == 0) *n_steps_sm = nsteps;
      __syncwarp();
      mbar_arrive(bar_steps);  // release: every lane's table writes
    }
    // ---------------------------------------------- K box 0 / box 1, V copies
    // K: one warp per (box, step parity); a K stage is only ever reused by
    // steps of one parity (KS is even), so each warp's ring waits are in
    // order.  V: one warp per box over every step, because a V stage is
    // reused by steps of both parities (VS is odd): a warp that skipped the
    // other parity's uses could test a ring barrier two phases behind.
    const bool is_k = warp <= 12;
    const int bx = is_k ? ((warp == 8 || warp == 10) ? 0 : 1) : warp - 14;
    const int par = is_k ? ((warp == 8 || warp == 11) ? 0 : 1) : 0;
    const int stride = is_k ? 2 : 1;
    if (lane == 0 && bx < C::KB) {
      if constexpr (!RASTER) tma_prefetch_desc(is_k ? &maps.k : &maps.v);
      const int RS = is_k ? KS : VS;
      bool ok = mbar_wait(bar_steps, 0, abort_flag);
      const int n = ok ? *n_steps_sm : 0;
      int j = par;
      for (; ok && j < n; j += stride) {
        const int s = j % RS;
        const uint32_t emp = is_k ? kempty(s) : vempty(s);
        const uint32_t ful = is_k ? kfull(s) : vfull(s);
        if (j >= RS && !mbar_wait(emp, ((j / RS) - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        const int t = int(steps[j] & kTileMask);
        // box bx of the block: [box][row][64] in the stage
        mbar_arrive_expect_tx(ful, C::BOX);
        kv_copy<D, RASTER>(is_k ? sK + (bx * KS + s) * C::BOX : sV + s * C::BLK_BYTES + bx * C::BOX,
                           maps, is_k, ful, bx, t, bh, g, io.codes);
      }
      if (!ok) report_timeout(abort_flag, status);
      // On any abort (this warp's own wait or another role's), the consumers
      // may have quit before reading this warp's last copies: wait, bounded,
      // for the ones that can still be in flight, its last uses of the ring
      // (RS steps back: 4 stages of one parity for K, 5 for V), so that no
      // copy writes shared memory after the CTA has moved on.
      if (!ok || *abort_flag) {
        for (int jj = j - stride; jj >= 0 && jj >= j - RS; jj -= stride)
          mbar_wait(ful_of(is_k, jj % RS), (jj / RS) & 1, nullptr, 200000000ull);
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ score bursts
    if (lane == 0) {
      constexpr uint32_t idesc_qk2 = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t idesc_qk1 = idesc_bf16_f32(128, 64, false);
      bool ok = mbar_wait(bar_qready, 0, abort_flag) && mbar_wait(bar_steps, 0, abort_flag);
      const int n = ok ? *n_steps_sm : 0;
      // pair t: scores of steps 2t and 2t+1 into S0 | S1 (adjacent TMEM
      // columns); needs K of both steps and both groups done reading the
      // previous pair's S.  An odd last step gets an N=64 burst of its own.
      for (int t = 0; ok && 2 * t < n; ++t) {
        const int j0 = 2 * t, s0 = j0 % KS;
        const bool two = j0 + 1 < n;
        // K normally lands long before the groups free S: wait for it first
        ok = mbar_wait(kfull(s0), (j0 / KS) & 1, abort_flag) &&
             (!two || mbar_wait(kfull(s0 + 1), ((j0 + 1) / KS) & 1, abort_flag));
        if (ok && t > 0) ok = mbar_wait(bar_sfree, (t - 1) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t bd =
              sdesc_sw128(sK + ((kk / 4) * KS + s0) * C::BOX + (kk % 4) * 32, 16, 1024);
          tc_mma_ts(tmem + C::COL_S, tmem + C::COL_Q + 8u * kk, bd, two ? idesc_qk2 : idesc_qk1,
                    kk > 0 ? 1u : 0u);
        }
        tc_commit(bar_s);
        tc_commit(kempty(s0));
        if (two) tc_commit(kempty(s0 + 1));
      }
      if (!ok) report_timeout(abort_flag, status);
      // every MMA this thread issued has completed once its drain barrier flips
      tc_commit(bar_drain);
      mbar_wait(bar_drain, 0, nullptr, 200000000ull);
    }
    __syncwarp();
  } else if (warp == 13) {
    // ------------------------------------------------------------ PV issuer
    // PVs in step order (groups alternate): PV_j needs P_j and V_j.  The
    // order matters for the V ring: a stage is reused every VS steps by
    // both groups, and testing its barrier for step j is unambiguous only
    // once PV_{j-VS} has been issued.
    if (lane == 0) {
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, true);
      bool ok = mbar_wait(bar_steps, 0, abort_flag);
      // test hook: with stall_pv set no PV is issued, so the softmax's wait
      // on the first PV runs out and the kernel takes its timeout path
      const int n = ok && !g.stall_pv ? *n_steps_sm : 0;
      for (int j = 0; ok && j < n; ++j) {
        const int w = j & 1, s = j % VS;
        ok = mbar_wait(vfull(s), (j / VS) & 1, abort_flag) &&
             mbar_wait(bar_p + 8 * w, (j >> 1) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t bd = sdesc_sw128(sV + s * C::BLK_BYTES + kk * 2048, C::BOX, 1024);
          tc_mma_ts(tmem + C::COL_O + 128u * w, tmem + C::COL_P + 32u * w + 8u * kk, bd,
                    idesc_pv, (j >= 2 || kk > 0) ? 1u : 0u);
        }
        tc_commit(bar_o + 8 * w);
        tc_commit(vempty(s));
      }
      if (!ok) report_timeout(abort_flag, status);
      tc_commit(bar_drain + 8);
      mbar_wait(bar_drain + 8, 0, nullptr, 200000000ull);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int wg = warp >> 2, quad = warp & 3;
    const int row = quad * 32 + lane;
    const int half = quad >> 1;
    const int qb = 2 * pair + half;
    const uint32_t lane_base = uint32_t(quad * 32) << 16;
    const bool q_exists = qb < g.nb;
    const bool row_valid =
        q_exists && ((__ldg(bmask + int64_t(b) * g.nb + qb) >> (row & 63)) & 1ull);
    bool ok = true;

    if (wg == 0) {
      // Q rows into tensor memory (A operand of S = Q K^T), bf16 pairs per column
      uint32_t qr[D / 2];
      const int64_t qrow = int64_t(pair) * 128 + row;
      const __nv_bfloat16* qsrc = nullptr;
      if (qrow < g.N) {
        if constexpr (RASTER) {
          // the slot's raster token; pad slots read nothing (their rows are
          // zero and their outputs are written as 0)
          const uint32_t pr = uint32_t(__ldg(io.perm + int64_t(b) * g.N + qrow));
          if (!(pr & 0x80000000u))
            qsrc = io.q + int64_t(b) * io.qsb + int64_t(pr) * io.qsn + int64_t(bh - b * g.h) * io.qsh;
        } else {
          qsrc = io.q + (int64_t(bh) * g.N + qrow) * D;
        }
      }
      if (qsrc) {
        const uint4* src = reinterpret_cast<const uint4*>(qsrc);
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
          const uint4 u = __ldg(src + i);
          qr[4 * i] = u.x;
          qr[4 * i + 1] = u.y;
          qr[4 * i + 2] = u.z;
          qr[4 * i + 3] = u.w;
        }
      } else {
#pragma unroll
        for (int i = 0; i < D / 2; ++i) qr[i] = 0u;
      }
      if constexpr (D == 128) {
        BSA_TMEM_ST64(tmem + C::COL_Q + lane_base, qr);
      } else {
        BSA_TMEM_ST32(tmem + C::COL_Q + lane_base, qr);
      }
      tc_fence_before();
      mbar_arrive(bar_qready);
    }

    const uint32_t tS = tmem + C::COL_S + 64u * wg + lane_base;
    const uint32_t tP = tmem + C::COL_P + 32u * wg + lane_base;
    const uint32_t tO = tmem + C::COL_O + 128u * wg + lane_base;
    const float sl2 = g.scale * 1.4426950408889634f;
    float m_used = -INFINITY, l_sum = 0.f;
    int k = 0;  // steps of this group so far
    // this group's steps are every other entry of the step table.  Barrier
    // probes are issued ahead of independent work so that their latency
    // (~170 cycles even for a completed phase) overlaps it.
    // window heads: this row's grid coordinates and its head's window
    struct {
      bool video;
      int tq, yq, xq, wt, wy, wx;
    } win = {false, 0, 0, 0, -1, -1, -1};
    if constexpr (MODE == kModeWindow) {
      if (q_exists && qb >= g.nbp) {
        const int v = int(uint32_t(__ldg(io.perm + int64_t(b) * g.N + int64_t(qb) * 64 +
                                         (row & 63))) & 0x7FFFFFFFu) - g.P;
        const int hw = g.H * g.W;
        win.video = true;
        win.tq = v / hw;
        win.yq = (v - win.tq * hw) / g.W;
        win.xq = v - win.tq * hw - win.yq * g.W;
        const int32_t* w3 = io.windows + 3 * (bh - b * g.h);
        win.wt = __ldg(w3);
        win.wy = __ldg(w3 + 1);
        win.wx = __ldg(w3 + 2);
      }
    }
    ok = __all_sync(0xffffffffu, mbar_wait(bar_steps, 0, abort_flag));
    const int n = ok ? *n_steps_sm : 0;
    const uint64_t* bm_row = bmask + int64_t(b) * g.nb;
    // s_next: the next pair's S was ready when probed after this step's
    // exponentials (a completed phase stays completed until this group
    // frees S again)
    bool s_next = false;
    for (int j = wg; ok && j < n; j += 2, ++k) {
      const bool s_ready = __all_sync(0xffffffffu, s_next || mbar_test(bar_s, k & 1));
      const uint32_t entry = steps[j];
      const int tile = int(entry & kTileMask);
      const uint32_t flags = entry >> kFlagShift;
      const bool member = (flags >> half) & 1u;
      if (!s_ready) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar_s, k & 1, abort_flag));
        if (!ok) break;
      }
      tc_fence_after();
      uint32_t pk[32];
      float factor = 1.f;
      bool rescale = false;
      bool o_ready = k == 0;
      if (member) {
        uint32_t r[64];
        BSA_TMEM_LD64(tS, r);
        tc_fence_before();
        mbar_arrive(bar_sfree);
        bool all_valid = (flags & 4u) != 0u;
        uint64_t vm = all_valid ? ~0ull : __ldg(bm_row + tile);
        if constexpr (MODE == kModeWindow) {
          // the row's element mask for this key block (boundary tiles);
          // prefix rows and prefix keys are dense
          if (win.video && tile >= g.nbp) {
            Box kx;
            video_block_box(g, io.codes, b, tile, kx);
            vm &= window_bits(kx, win.tq, win.yq, win.xq, win.wt, win.wy, win.wx);
          }
          all_valid = __all_sync(0xffffffffu, vm == ~0ull);
        }
        const uint32_t lo = uint32_t(vm), hi = uint32_t(vm >> 32);
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        if (all_valid) {
#pragma unroll
          for (int c = 0; c < 64; c += 2)
            mx[(c >> 1) & 3] =
                max3f(mx[(c >> 1) & 3], __uint_as_float(r[c]), __uint_as_float(r[c + 1]));
        } else {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (bit_of(lo, hi, c)) mx[c & 3] = fmaxf(mx[c & 3], __uint_as_float(r[c]));
        }
        const float mxs = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * sl2;
        if (mxs > m_used + 8.f) {
          if (m_used != -INFINITY) {
            factor = ex2_approx(m_used - mxs);
            rescale = true;
          }
          m_used = mxs;
        }
        float sum[4] = {0.f, 0.f, 0.f, 0.f};
        // the previous PV of this group: probed halfway through the
        // exponentials, the answer used after them
        bool o_probe = true;
        if (all_valid) {
          // two columns per instruction for the scaling and the row sum
#pragma unroll
          for (int c = 0; c < 64; c += 2) {
            if (c == 32 && k > 0) o_probe = mbar_test_after(bar_o + 8 * wg, (k - 1) & 1, sum[0]);
            float x0, x1;
            fma_f32x2(x0, x1, __uint_as_float(r[c]), __uint_as_float(r[c + 1]), sl2, sl2, -m_used,
                      -m_used);
            // one column pair in four on the FMA pipe, the rest on MUFU
            float p0, p1;
            if (((c >> 1) & 3) == 3) {
              exp2_poly_x2(p0, p1, x0, x1);
            } else {
              p0 = ex2_approx(x0);
              p1 = ex2_approx(x1);
            }
            const int a = (c >> 1) & 1;
            add_f32x2(sum[2 * a], sum[2 * a + 1], sum[2 * a], sum[2 * a + 1], p0, p1);
            pk[c / 2] = pack_bf16x2(p0, p1);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 64; c += 2) {
            if (c == 32 && k > 0) o_probe = mbar_test_after(bar_o + 8 * wg, (k - 1) & 1, sum[0]);
            const float p0 =
                bit_of(lo, hi, c) ? ex2_approx(fmaf(__uint_as_float(r[c]), sl2, -m_used)) : 0.f;
            const float p1 = bit_of(lo, hi, c + 1)
                                 ? ex2_approx(fmaf(__uint_as_float(r[c + 1]), sl2, -m_used))
                                 : 0.f;
            sum[(c >> 1) & 3] += p0 + p1;
            pk[c / 2] = pack_bf16x2(p0, p1);
          }
        }
        l_sum = l_sum * factor + ((sum[0] + sum[1]) + (sum[2] + sum[3]));
        s_next = mbar_test_after(bar_s, (k + 1) & 1, l_sum);
        o_ready = __all_sync(0xffffffffu, o_probe);
      } else {
        s_next = false;
        tc_fence_before();
        mbar_arrive(bar_sfree);
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = 0u;
      }
      // P and O of this group are free once its previous PV has finished
      if (!o_ready) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar_o + 8 * wg, (k - 1) & 1, abort_flag));
        if (!ok) break;
      }
      tc_fence_after();
      if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t o[32];
          BSA_TMEM_LD32(tO + 32u * ch, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * factor);
          BSA_TMEM_ST32(tO + 32u * ch, o);
        }
      }
      BSA_TMEM_ST32(tP, pk);
      tc_fence_before();
      mbar_arrive(bar_p + 8 * wg);
    }
    // ---------------------------------------------------------- epilogue
    if (ok && k > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar_o + 8 * wg, (k - 1) & 1, abort_flag));
    xch[wg * 128 + row] = m_used;
    xch[256 + wg * 128 + row] = l_sum;
    named_bar_sync(1, 256);
    ok = ok && !*abort_flag;
    if (!ok) {
      if (lane == 0) report_timeout(abort_flag, status);
    } else if (q_exists) {
      tc_fence_after();
      const float m0 = xch[row], m1 = xch[128 + row];
      const float l0 = xch[256 + row], l1 = xch[384 + row];
      const float m = fmaxf(m0, m1);
      const float a0 = (m0 == -INFINITY) ? 0.f : ex2_approx(m0 - m);
      const float a1 = (m1 == -INFINITY) ? 0.f : ex2_approx(m1 - m);
      const float l = l0 * a0 + l1 * a1;
      const float inv = (row_valid && l > 0.f) ? 1.f / l : 0.f;
      const float f0 = a0 * inv, f1 = a1 * inv;
      // the row's log-sum-exp in the exp2 domain, for the backward
      // (P = exp2(s * scale * log2(e) - lse2)); +inf for pad rows
      if (io.lse && wg == 0)
        io.lse[int64_t(bh) * g.N + int64_t(qb) * 64 + (row & 63)] =
            (row_valid && l > 0.f) ? m + __log2f(l) : INFINITY;
      __nv_bfloat16* orow;
      if constexpr (RASTER) {
        const int64_t slot = int64_t(qb) * 64 + (row & 63);
        const int64_t pr = int64_t(uint32_t(__ldg(io.perm + int64_t(b) * g.N + slot)) & 0x7FFFFFFFu);
        orow = io.o + int64_t(b) * io.osb + pr * io.osn + int64_t(bh - b * g.h) * io.osh;
      } else {
        orow = io.o + (int64_t(bh) * g.N + int64_t(qb) * 64 + (row & 63)) * D;
      }
      // group wg writes columns [wg*D/2, (wg+1)*D/2)
#pragma unroll
      for (int ch = 0; ch < D / 64; ++ch) {
        const uint32_t col = uint32_t(wg * (D / 2) + ch * 32);
        uint32_t o0[32], o1[32];
        BSA_TMEM_LD32(tmem + C::COL_O + col + lane_base, o0);
        BSA_TMEM_LD32(tmem + C::COL_O + 128u + col + lane_base, o1);
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float x0 = (a0 != 0.f ? __uint_as_float(o0[2 * i]) * f0 : 0.f) +
                           (a1 != 0.f ? __uint_as_float(o1[2 * i]) * f1 : 0.f);
          const float x1 = (a0 != 0.f ? __uint_as_float(o0[2 * i + 1]) * f0 : 0.f) +
                           (a1 != 0.f ? __uint_as_float(o1[2 * i + 1]) * f1 : 0.f);
          w[i] = pack_bf16x2(x0, x1);
        }
        uint4* dst = reinterpret_cast<uint4*>(orow + col);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int D, int MODE, bool RASTER>
cudaError_t launch_t(const Geo& g, const KVMaps<RASTER>& maps, const AttnIO& io, cudaStream_t st) {
  using C = Cfg<D>;
  auto kern = attn_fwd_kernel<D, MODE, RASTER>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid((g.nb + 1) / 2, g.B * g.h);
  kern<<<grid, C::kThreads, C::SMEM, st>>>(maps, g, io);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const Geo& g, const KVMaps<false>& maps, const AttnIO& io,
                             bool dense, cudaStream_t st) {
  if (g.d == 128)
    return dense ? launch_t<128, kModeDense, false>(g, maps, io, st)
                 : launch_t<128, kModeLists, false>(g, maps, io, st);
  return dense ? launch_t<64, kModeDense, false>(g, maps, io, st)
               : launch_t<64, kModeLists, false>(g, maps, io, st);
}

cudaError_t launch_attention_raster(const Geo& g, const KVMaps<true>& maps, const AttnIO& io,
                                    cudaStream_t st) {
  if (io.windows) {
    if (g.d == 128) return launch_t<128, kModeWindow, true>(g, maps, io, st);
    return launch_t<64, kModeWindow, true>(g, maps, io, st);
  }
  if (g.d == 128) return launch_t<128, kModeLists, true>(g, maps, io, st);
  return launch_t<64, kModeLists, true>(g, maps, io, st);
}

}  // namespace bsa
