// Block-sparse attention forward on sm_100a: TMA-fed tcgen05 tiles with the
// accumulators and the A operands in tensor memory, walking a per-query-block
// list of kept key blocks so that only kept 64x64 tiles are ever loaded or
// multiplied (Sparse VideoGen on TPU, aibase.it, section "이론적 sparsity와
// 물리적 sparsity의 차이": skipping empty tiles is where the speed comes
// from).
//
// CTA = two adjacent query blocks (128 query rows = the full tcgen05 M=128
// datapath; M=64 would leave half of it idle).  The two blocks' sorted key
// lists are merged on the fly into a sequence of steps, one 64-token key
// block each.  Steps go in pairs (one per softmax warpgroup) and each pair's
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
//
// Two softmax warpgroups take alternate steps, each with its own running
// max, running sum and O accumulator (an exact split of the key set); the
// epilogue merges them: O = (a0*O0 + a1*O1) / (a0*l0 + a1*l1),
// a_w = 2^(m_w - max(m0, m1)).  The softmax is the exact online softmax in
// the exp2 domain with a lazily updated running max: O is rescaled only
// when the row max grows by more than 8 (so every probability stays below
// 2^8), which is still exact after the final division.
//
// Warp roles (512 threads):
//   warps 0-3 / 4-7  softmax warpgroup 0 / 1; thread r of a group owns
//                    query row r = TMEM lane r (warp w reaches lanes
//                    32*(w%4)..+31); group 0 first copies Q into TMEM
//   warp 8           stages the index lists, merges them, publishes each
//                    step, and copies box 0 (head_dim 0-63) of even steps' K
//   warp 9           TMEM allocator; one thread issues the score bursts
//   warp 10          K box 0 of odd steps
//   warps 11 / 12    K box 1 (head_dim 64-127) of even / odd steps
//   warp 13          one thread issues the PV MMAs of both softmax groups
//   warps 14 / 15    V of even / odd steps (both halves in one copy)
// One issuing thread completes about one bulk tensor copy per ~650 cycles
// whatever its size, so copies are spread over six warps and V moves as a
// single 16 KB copy; tcgen05.mma blocks its issuing thread while the tensor
// pipe is busy, so score bursts and PVs come from two threads.
// Tensor memory (512 columns): Q [0,64) bf16 pairs | S0 [64,128) | S1
// [128,192) | P0 [192,224) | P1 [224,256) | O0 [256,384) | O1 [384,512).
//
// Every wait is bounded (2 s); a timeout sets the caller's status word to
// BSA_ERR_TIMEOUT, drains in-flight copies and MMAs and frees tensor memory.
#include <climits>

#include "bsa_internal.cuh"

namespace bsa {
namespace {

template <int D>
struct Cfg {
  static constexpr int kThreads = 512;
  static constexpr int KB = D / 64;  // 64-column boxes per block (copy streams per ring)
  static constexpr int KS = 8;                    // K ring stages (even: pairs)
  static constexpr int VS = 5;                    // V ring stages
  static constexpr int IR = 16;                   // step-info ring entries
  static constexpr int BLK_BYTES = 64 * D * 2;    // one K (or V) block
  static constexpr int BOX = 64 * 128;            // one 64-column TMA box of a block
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_Q = 0, COL_S = 64, COL_P = 192, COL_O = 256;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = KS * BLK_BYTES;
  static constexpr int OFF_BAR = OFF_V + VS * BLK_BYTES;
  // kfull[KS] kempty[KS] vfull[VS] vempty[VS] qready s sfree[2] p[2] o[2] drain[2]
  static constexpr int N_BARS = 2 * KS + 2 * VS + 11;
  static constexpr int OFF_INFO = OFF_BAR + 8 * N_BARS;
  static constexpr int OFF_XCH = OFF_INFO + 24 * IR;  // float m[2][128], l[2][128]
  static constexpr int LIST_CAP = 1024;  // index-list entries cached per query block
  static constexpr int FULL_CAP = 2560;  // blocks whose full/partial byte is cached
  static constexpr int OFF_LIST = OFF_XCH + 4 * 4 * 128;
  static constexpr int OFF_FULL = OFF_LIST + 2 * 4 * LIST_CAP;
  static constexpr int OFF_MISC = OFF_FULL + FULL_CAP;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;  // + slack for 1024-B alignment
  static_assert(KS % 2 == 0, "step pairs must not straddle the K ring's end");
  // A step's info entry is overwritten only after the score burst of the
  // step KS later has run, which needs both groups past step j+KS-2.
  static_assert(IR > KS + 2 && IR <= 32, "step-info ring size");
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

struct StepInfo {
  int32_t tag;     // j+1 once the entry describes step j (0 = none yet)
  int32_t tile;    // key block, or -1 = no more steps
  uint32_t flags;  // bit 0: first query block keeps it; bit 1: second one
  uint32_t pad;
  uint64_t vmask;  // valid-slot mask of the key block
};
static_assert(sizeof(StepInfo) == 24, "StepInfo layout");

// Iterator over the kept key blocks of one query block, in rotated order:
// blocks >= `start` ascending, then the blocks below `start` ascending.
// CTAs working on the same head start at different blocks, so they do not
// all fetch the same K/V tiles at the same moment (the online softmax does
// not depend on the order of its steps).  p points to the shared-memory
// copy of the list, or to global memory for very long lists; a dense row
// walks every block.  peek() returns the rotated key (block - start) mod nb
// of the next block, INT_MAX when done.
struct ListIt {
  const int32_t* p;
  int n;       // list length (every block for a dense row)
  bool dense;
  int first;   // position of the first block >= start
  int taken;   // blocks handed out so far
  int start, nb;
  __device__ void init(int start_, int nb_) {
    start = start_;
    nb = nb_;
    taken = 0;
    if (dense) {
      first = start;
      return;
    }
    int lo = 0, hi = n;  // lower_bound(p, p+n, start)
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (p[mid] < start) lo = mid + 1; else hi = mid;
    }
    first = lo;
  }
  __device__ int block_at(int i) const { return dense ? i : p[i]; }
  __device__ int peek() const {
    if (taken >= n) return INT_MAX;
    int i = first + taken;
    if (i >= n) i -= n;
    const int v = block_at(i);
    return v >= start ? v - start : v + nb - start;
  }
};

__device__ __forceinline__ void report_timeout(volatile int* abort_flag, int32_t* status) {
  *abort_flag = 1;
  atomicCAS(status, 0, int32_t(BSA_ERR_TIMEOUT));
}

__device__ __forceinline__ bool bit_of(uint32_t lo, uint32_t hi, int c) {
  return ((c < 32 ? (lo >> c) : (hi >> (c - 32))) & 1u) != 0u;
}

// Idle bookkeeping for the polling loops: expired() turns true once no
// progress was made for 2 s or another role has aborted.
struct IdleClock {
  uint32_t idle = 0;
  uint64_t since = 0;
  __device__ void progress() { idle = 0; }
  __device__ bool expired(volatile int* abort_flag) {
    if ((++idle & 255) != 0) return false;
    const uint64_t now = global_timer_ns();
    if (idle == 256) since = now;
    return *abort_flag || now - since > 2000000000ull;
  }
};

template <int D, bool DENSE>
__global__ void __launch_bounds__(512, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap mk, const __grid_constant__ CUtensorMap mv,
                    Geo g, const __nv_bfloat16* __restrict__ qperm,
                    const uint64_t* __restrict__ bmask, const uint8_t* __restrict__ bfull,
                    const int32_t* __restrict__ idx, const int32_t* __restrict__ cnt,
                    __nv_bfloat16* __restrict__ out, int32_t* __restrict__ status) {
  using C = Cfg<D>;
  constexpr int KS = C::KS, VS = C::VS, IR = C::IR;
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
  const uint32_t bar_sfree = bar_qready + 16;  // [2] group w has read its S (128 arrivals)
  const uint32_t bar_p = bar_qready + 32;      // [2] P written + O corrected (128 arrivals)
  const uint32_t bar_o = bar_qready + 48;      // [2] PV of group w finished
  const uint32_t bar_drain = bar_qready + 64;  // [2] score issuer, PV issuer
  StepInfo* info = reinterpret_cast<StepInfo*>(sm + C::OFF_INFO);
  float* xch = reinterpret_cast<float*>(sm + C::OFF_XCH);  // m[2][128] then l[2][128]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x, bh = blockIdx.y, b = bh / g.h;

  if (threadIdx.x == 0) {
    for (int s = 0; s < KS; ++s) {
      mbar_init(kfull(s), C::KB);
      mbar_init(kempty(s), 1);
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(vfull(s), 1);
      mbar_init(vempty(s), 1);
    }
    mbar_init(bar_qready, 128);
    mbar_init(bar_s, 1);
    for (int w = 0; w < 2; ++w) {
      mbar_init(bar_sfree + 8 * w, 128);
      mbar_init(bar_p + 8 * w, 128);
      mbar_init(bar_o + 8 * w, 1);
    }
    mbar_init(bar_drain, 1);
    mbar_init(bar_drain + 8, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 8 && lane < IR) info[lane].tag = 0;
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 8) {
    // ---------------------------------------------- list merge + K box 0
    // The whole warp stages both index lists and the per-block "all slots
    // valid" bytes in shared memory; lane 0 then merges the lists, publishes
    // step j once K stage j%KS is free (so an info entry is never reused
    // before every reader is past it) and copies box 0 of K_j.  After the
    // last step it publishes two end markers (steps n and n+1).
    int32_t* slist = reinterpret_cast<int32_t*>(sm + C::OFF_LIST);
    uint8_t* sfull = sm + C::OFF_FULL;
    const bool full_cached = g.nb <= C::FULL_CAP;
    const uint8_t* gfull = bfull + int64_t(b) * g.nb;
    if (full_cached)
      for (int i = lane; i < g.nb; i += 32) sfull[i] = __ldg(gfull + i);
    ListIt it[2];
    for (int hf = 0; hf < 2; ++hf) {
      const int qb = 2 * pair + hf;
      it[hf].p = nullptr;
      it[hf].n = 0;
      it[hf].dense = false;
      if (qb < g.nb) {
        const int c = DENSE ? -1 : __ldg(cnt + int64_t(bh) * g.nb + qb);
        if (c < 0) {
          it[hf].dense = true;
          it[hf].n = g.nb;
        } else {
          const int32_t* src = idx + (int64_t(bh) * g.nb + qb) * g.kcap;
          it[hf].n = c;
          if (c <= C::LIST_CAP) {
            for (int i = lane; i < c; i += 32) slist[hf * C::LIST_CAP + i] = __ldg(src + i);
            it[hf].p = slist + hf * C::LIST_CAP;
          } else {
            it[hf].p = src;
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) {
      tma_prefetch_desc(&mk);
      tma_prefetch_desc(&mv);
      const int start = int((uint32_t(pair) * 61u + uint32_t(bh) * 17u) % uint32_t(g.nb));
      it[0].init(start, g.nb);
      it[1].init(start, g.nb);
      int j = 0, ends = 0;
      bool ok = true;
      for (;; ++j) {
        const int s = j % KS;
        if (j >= KS && !mbar_wait(kempty(s), ((j / KS) - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        StepInfo& e = info[j % IR];
        int t = INT_MAX;
        if (ends == 0) {
          const int ra = it[0].peek(), rb = it[1].peek();
          const int r = ra < rb ? ra : rb;
          if (r != INT_MAX) {
            t = r + start < g.nb ? r + start : r + start - g.nb;
            uint32_t flags = 0;
            if (ra == r) { flags |= 1u; ++it[0].taken; }
            if (rb == r) { flags |= 2u; ++it[1].taken; }
            const bool whole = full_cached ? (sfull[t] != 0) : (__ldg(gfull + t) != 0);
            e.tile = t;
            e.flags = flags;
            e.vmask = whole ? ~0ull : __ldg(bmask + int64_t(b) * g.nb + t);
          }
        }
        if (t == INT_MAX) e.tile = -1;
        __threadfence_block();
        *reinterpret_cast<volatile int32_t*>(&e.tag) = j + 1;
        if ((j & 1) == 0) {  // K box 0 of even steps
          if (t == INT_MAX) {
            mbar_arrive(kfull(s));
          } else {
            mbar_arrive_expect_tx(kfull(s), C::BOX);
            tma_load_3d(sK + s * C::BOX, &mk, kfull(s), 0, t * 64, bh);
          }
        }
        if (t == INT_MAX && ++ends == 2) break;
      }
      if (!ok) {
        report_timeout(abort_flag, status);
        for (int jj = j - 1; jj >= 0 && jj >= j - KS; --jj)
          mbar_wait(kfull(jj % KS), (jj / KS) & 1, nullptr, 200000000ull);
      }
    }
    __syncwarp();
  } else if (warp == 10 || warp == 11 || warp == 12 || warp == 14 || warp == 15) {
    // ---------------------------------------------- K box 0 odd, K box 1, V
    const bool is_k = warp <= 12;
    const int bx = warp == 10 ? 0 : 1;        // K box (unused for V)
    const int par = (warp == 11 || warp == 14) ? 0 : 1;
    if (lane == 0 && (!is_k || bx < C::KB)) {
      const int RS = is_k ? KS : VS;
      int j = par;
      bool ok = true;
      for (;; j += 2) {
        // sleep on the ring first; the step is normally published by then
        const int s = j % RS;
        const uint32_t emp = is_k ? kempty(s) : vempty(s);
        const uint32_t ful = is_k ? kfull(s) : vfull(s);
        if (j >= RS && !mbar_wait(emp, ((j / RS) - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        const StepInfo& e = info[j % IR];
        {
          bool seen = false;
          IdleClock clk;
          for (;;) {
            seen = *reinterpret_cast<const volatile int32_t*>(&e.tag) == j + 1;
            if (seen || clk.expired(abort_flag)) break;
          }
          if (!seen) {
            ok = false;
            break;
          }
        }
        __threadfence_block();
        const int t = *reinterpret_cast<const volatile int32_t*>(&e.tile);
        if (t < 0) {  // each parity meets exactly one of the two end markers
          if (is_k) mbar_arrive(ful);
          break;
        }
        if (is_k) {
          mbar_arrive_expect_tx(ful, C::BOX);
          tma_load_3d(sK + (bx * KS + s) * C::BOX, &mk, ful, 64 * bx, t * 64, bh);
        } else {
          mbar_arrive_expect_tx(ful, C::BLK_BYTES);
          if constexpr (D == 128)
            tma_load_4d(sV + s * C::BLK_BYTES, &mv, ful, 0, t * 64, 0, bh);
          else
            tma_load_3d(sV + s * C::BLK_BYTES, &mv, ful, 0, t * 64, bh);
        }
      }
      if (!ok) {
        report_timeout(abort_flag, status);
        for (int jj = j - 2; jj >= 0 && jj >= j - 2 * RS; jj -= 2)
          mbar_wait(ful_of(is_k, jj % RS), (jj / RS) & 1, nullptr, 200000000ull);
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ score bursts
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false);
      bool ok = mbar_wait(bar_qready, 0, abort_flag);
      // pair t: scores of steps 2t and 2t+1 into S0 | S1 (adjacent TMEM
      // columns); needs K of both steps and both groups done reading the
      // previous pair's S
      for (int t = 0; ok; ++t) {
        const int j0 = 2 * t, s0 = j0 % KS;
        if (t > 0) ok = mbar_wait(bar_sfree, (t - 1) & 1, abort_flag) &&
                        mbar_wait(bar_sfree + 8, (t - 1) & 1, abort_flag);
        if (ok) ok = mbar_wait(kfull(s0), (j0 / KS) & 1, abort_flag) &&
                     mbar_wait(kfull(s0 + 1), ((j0 + 1) / KS) & 1, abort_flag);
        if (!ok) break;
        if (*reinterpret_cast<volatile int32_t*>(&info[j0 % IR].tile) < 0) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t bd =
              sdesc_sw128(sK + ((kk / 4) * KS + s0) * C::BOX + (kk % 4) * 32, 16, 1024);
          tc_mma_ts(tmem + C::COL_S, tmem + C::COL_Q + 8u * kk, bd, idesc_qk, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar_s);
        tc_commit(kempty(s0));
        tc_commit(kempty(s0 + 1));
        if (*reinterpret_cast<volatile int32_t*>(&info[(j0 + 1) % IR].tile) < 0) break;
      }
      if (!ok) report_timeout(abort_flag, status);
      // every MMA this thread issued has completed once its drain barrier flips
      tc_commit(bar_drain);
      mbar_wait(bar_drain, 0, nullptr, 200000000ull);
    }
    __syncwarp();
  } else if (warp == 13) {
    // ------------------------------------------------------------ PV issuer
    // Two independent queues (one per softmax group), served in whichever
    // order they become ready: PV_j needs P_j and V_j.  A group is done at
    // its first end marker.
    if (lane == 0) {
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, true);
      int jp[2] = {0, 1};
      bool done[2] = {false, false};
      bool ok = true;
      IdleClock clk;
      while (ok && !(done[0] && done[1])) {
        bool progress = false;
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          if (done[w]) continue;
          const int j = jp[w];
          const StepInfo& e = info[j % IR];
          if (*reinterpret_cast<const volatile int32_t*>(&e.tag) != j + 1) continue;
          __threadfence_block();
          if (*reinterpret_cast<const volatile int32_t*>(&e.tile) < 0) {
            done[w] = true;
            progress = true;
            continue;
          }
          const int s = j % VS;
          if (!mbar_test(bar_p + 8 * w, (j >> 1) & 1) || !mbar_test(vfull(s), (j / VS) & 1))
            continue;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bd = sdesc_sw128(sV + s * C::BLK_BYTES + kk * 2048, C::BOX, 1024);
            tc_mma_ts(tmem + C::COL_O + 128u * w, tmem + C::COL_P + 32u * w + 8u * kk, bd,
                      idesc_pv, (j >= 2 || kk > 0) ? 1u : 0u);
          }
          tc_commit(bar_o + 8 * w);
          tc_commit(vempty(s));
          jp[w] = j + 2;
          progress = true;
        }
        if (progress)
          clk.progress();
        else if (clk.expired(abort_flag))
          ok = false;
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
      if (qrow < g.N) {
        const uint4* src = reinterpret_cast<const uint4*>(qperm + (int64_t(bh) * g.N + qrow) * D);
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
    for (int j = wg;; j += 2, ++k) {
      // the producer publishes step j's info (tag j+1) before its K copy
      const StepInfo& e = info[j % IR];
      {
        bool seen = false;
        IdleClock clk;
        for (;;) {
          seen = *reinterpret_cast<const volatile int32_t*>(&e.tag) == j + 1;
          if (seen || clk.expired(abort_flag)) break;
        }
        ok = __all_sync(0xffffffffu, seen);
        if (!ok) break;
      }
      __threadfence_block();
      if (*reinterpret_cast<const volatile int32_t*>(&e.tile) < 0) break;
      const uint32_t flags = *reinterpret_cast<const volatile uint32_t*>(&e.flags);
      const uint64_t vm = *reinterpret_cast<const volatile uint64_t*>(&e.vmask);
      const bool member = (flags >> half) & 1u;
      ok = __all_sync(0xffffffffu, mbar_wait(bar_s, k & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      uint32_t pk[32];
      float factor = 1.f;
      bool rescale = false;
      if (member) {
        uint32_t r[64];
        BSA_TMEM_LD64(tS, r);
        tc_fence_before();
        mbar_arrive(bar_sfree + 8 * wg);
        const uint32_t lo = uint32_t(vm), hi = uint32_t(vm >> 32);
        const bool all_valid = (lo & hi) == 0xFFFFFFFFu;
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        if (all_valid) {
#pragma unroll
          for (int c = 0; c < 64; ++c) mx[c & 3] = fmaxf(mx[c & 3], __uint_as_float(r[c]));
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
        if (all_valid) {
#pragma unroll
          for (int c = 0; c < 64; c += 2) {
            const float p0 = ex2_approx(fmaf(__uint_as_float(r[c]), sl2, -m_used));
            const float p1 = ex2_approx(fmaf(__uint_as_float(r[c + 1]), sl2, -m_used));
            sum[(c >> 1) & 3] += p0 + p1;
            pk[c / 2] = pack_bf16x2(p0, p1);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 64; c += 2) {
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
      } else {
        tc_fence_before();
        mbar_arrive(bar_sfree + 8 * wg);
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = 0u;
      }
      // P and O of this group are free once its previous PV has finished
      if (k > 0) {
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
      __nv_bfloat16* orow = out + (int64_t(bh) * g.N + int64_t(qb) * 64 + (row & 63)) * D;
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

template <int D, bool DENSE>
cudaError_t launch_t(const Geo& g, LayoutPtrs lp, const CUtensorMap* maps,
                     const __nv_bfloat16* qp, const int32_t* idx, const int32_t* cnt,
                     __nv_bfloat16* o, int32_t* status, cudaStream_t st) {
  using C = Cfg<D>;
  auto kern = attn_fwd_kernel<D, DENSE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid((g.nb + 1) / 2, g.B * g.h);
  kern<<<grid, C::kThreads, C::SMEM, st>>>(maps[0], maps[1], g, qp, lp.bmask, lp.bfull, idx, cnt, o,
                                           status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const Geo& g, LayoutPtrs lp, const CUtensorMap* maps,
                             const __nv_bfloat16* qp, const int32_t* idx, const int32_t* cnt,
                             __nv_bfloat16* o, int32_t* dev_status, bool dense, cudaStream_t st) {
  if (g.d == 128)
    return dense ? launch_t<128, true>(g, lp, maps, qp, idx, cnt, o, dev_status, st)
                 : launch_t<128, false>(g, lp, maps, qp, idx, cnt, o, dev_status, st);
  return dense ? launch_t<64, true>(g, lp, maps, qp, idx, cnt, o, dev_status, st)
               : launch_t<64, false>(g, lp, maps, qp, idx, cnt, o, dev_status, st);
}

}  // namespace bsa
