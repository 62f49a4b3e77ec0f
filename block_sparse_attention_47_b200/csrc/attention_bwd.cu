// Backward of the block-sparse attention on sm_100a: gradients dQ, dK, dV
// over the same kept 64x64 tiles as the forward (Prism / Kandinsky 6 speed
// ablation, oh-my-gpu.com, section "같은 계산량 안에서 볼 곳을 고르는 Prism":
// the sparse attention also trains, a 2K step going from 26.5 to 10.6
// minutes).  With P = exp2(S * scale * log2(e) - lse2) recomputed from the
// forward's per-row log-sum-exp (exp2 domain) and D = rowsum(dO * O):
//     dP = dO V^T,  dS = P * (dP - D),
//     dQ = scale * dS K,  dK = scale * dS^T Q,  dV = P^T dO.
//
// Two kernels, both tcgen05 with the accumulators in tensor memory and the
// tiles in 128-byte-swizzled shared memory:
//   dQ   CTA = two adjacent query blocks (128 rows, as the forward), walking
//        the union of their key lists; per step S and dP (two SS MMAs,
//        M=128 N=64), dS from them in registers, then dQ += dS K (A = dS in
//        tensor memory, B = the same K tile read N-major).
//   dKdV CTA = two adjacent key blocks (128 key rows), walking the union of
//        the query blocks that kept them (transposed lists, built as
//        bitmaps); per step S^T = K Q^T and dP^T = V dO^T (M=128 N=64), P^T
//        and dS^T in registers, then dV += P^T dO and dK += dS^T Q.
// P needs no running maximum (the forward's statistics fix it), so steps
// are independent: two groups of row threads take alternate steps, each
// with its own S/dP columns in tensor memory, and one thread issues the
// copies and MMAs so that both groups compute while the tensor pipe runs:
//     iteration j:  the accumulation of step j-2, then S/dP of step j.
// Step tiles (K/V, or Q/dO with their rows' lse2 and D) go through a
// 4-stage ring loaded one step ahead.  P/dS are written over the group's
// own S and dP columns (in dQ, Q and dO sit in tensor memory as the A
// operands of S and dP; in dKdV the two accumulators fill the rest), so a
// group's next S/dP waits for its previous accumulation to finish.  Every wait is bounded (2 s) and reports
// BSA_ERR_TIMEOUT as the forward.
#include "bsa_internal.cuh"

namespace bsa {
namespace {

constexpr int kMaxWords = kAttnMaxBlocks / 32;
constexpr uint32_t kTileMask = 0x1FFFu, kFlagShift = 13;

template <int D>
struct BwdCfg {
  // warps 0-3 / 4-7: row groups 0 / 1 (alternate steps); 8: issuer; 9: steps
  static constexpr int kThreads = 320;
  static constexpr int KB = D / 64;                // 64-column boxes
  static constexpr int NS = 4;                     // step-tile ring stages
  static constexpr int TILE64 = 64 * D * 2;        // one 64-row tile
  static constexpr int TILE128 = 128 * D * 2;      // the CTA's own 128-row tile
  static constexpr int BOX64 = 64 * 128, BOX128 = 128 * 128;
  // dQ: own = Q | dO (128 rows each); stages = K | V (64 rows)
  // dKdV: own = K | V; stages = Q | dO, plus lse2 | delta (64 floats)
  static constexpr int OFF_OWN_A = 0;
  static constexpr int OFF_OWN_B = TILE128;
  static constexpr int OFF_STG = 2 * TILE128;              // [stage][a | b] 64-row tiles
  static constexpr int OFF_VEC = OFF_STG + NS * 2 * TILE64; // [stage][lse2 | delta][64] fp32
  static constexpr int OFF_BAR = OFF_VEC + NS * 2 * 64 * 4;
  // full[NS] empty[NS] s_ready[2] (spare[2]) x_ready[2] x_free[2] own steps done drain
  static constexpr int N_BARS = 2 * NS + 8 + 4;
  static constexpr int OFF_BM = OFF_BAR + 8 * N_BARS;      // uint32 A, B, F [kMaxWords]
  static constexpr int OFF_STEPS = OFF_BM + 3 * 4 * kMaxWords;
  static constexpr int OFF_MISC = OFF_STEPS + 2 * kAttnMaxBlocks;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  // tensor memory.  dQ: Q and dO (the A operands of S and dP, bf16 pairs) at
  // 0 and 64, group w's S at 128 + 128w (its dS written over it), dP 64
  // further, the accumulator at 384.  dKdV: group w's S at 128w (P^T over
  // it), dP at 128w + 64 (dS^T over it), dV at 256 and dK at 256 + D.
  static constexpr uint32_t COL_DQ_Q = 0, COL_DQ_DO = 64, COL_DQ_S = 128, COL_DQ_ACC = 384;
  static constexpr uint32_t COL_DV = 256, COL_DK = 256 + D;
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
  static_assert(COL_DK + D <= TMEM_COLS, "tensor memory budget");
};

struct BwdBars {
  uint32_t full, empty, s_ready, x_ready, x_free, own, steps, done, drain;
};

template <int D>
__device__ __forceinline__ BwdBars bwd_bars(uint32_t bar0) {
  using C = BwdCfg<D>;
  BwdBars b;
  b.full = bar0;
  b.empty = bar0 + 8 * C::NS;
  b.s_ready = bar0 + 16 * C::NS;
  b.x_ready = b.s_ready + 32;
  b.x_free = b.s_ready + 48;
  b.own = b.s_ready + 64;
  b.steps = b.own + 8;
  b.done = b.own + 16;
  b.drain = b.own + 24;
  return b;
}

template <int D>
__device__ __forceinline__ void bwd_init_bars(const BwdBars& b) {
  using C = BwdCfg<D>;
  for (int s = 0; s < C::NS; ++s) {
    mbar_init(b.full + 8 * s, 1);
    mbar_init(b.empty + 8 * s, 1);
  }
  for (int w = 0; w < 2; ++w) {
    mbar_init(b.s_ready + 8 * w, 1);
    mbar_init(b.x_ready + 8 * w, 128);
    mbar_init(b.x_free + 8 * w, 1);
  }
  mbar_init(b.own, 256);
  mbar_init(b.steps, 32);
  mbar_init(b.done, 1);
  mbar_init(b.drain, 1);
}

#define BSA_TMEM_ST16(taddr, r)                                                               \
  asm volatile(                                                                               \
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "                                        \
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n\t"                         \
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),                                          \
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), \
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),       \
      "r"(r[15])                                                                              \
      : "memory")

__device__ __forceinline__ void report_timeout(volatile int* abort_flag, int32_t* status) {
  *abort_flag = 1;
  atomicCAS(status, 0, int32_t(BSA_ERR_TIMEOUT));
}

__device__ __forceinline__ bool bit_of(uint32_t lo, uint32_t hi, int c) {
  return ((c < 32 ? (lo >> c) : (hi >> (c - 32))) & 1u) != 0u;
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

// The step table of one CTA (run by one warp): bitmaps A and B over the
// walked blocks, their union expanded in ascending order into 16-bit
// entries (block index, bit 13: A has it, bit 14: B has it, bit 15: the
// block is full).  Returns the number of steps (all lanes).
__device__ __forceinline__ int build_steps(const uint32_t* bmA, const uint32_t* bmB,
                                           const uint32_t* bmF, int nw, uint16_t* steps,
                                           int lane) {
  int nsteps = 0;
  for (int r0 = 0; r0 < nw; r0 += 32) {
    const int w = r0 + lane;
    const uint32_t a = w < nw ? bmA[w] : 0u, bb = w < nw ? bmB[w] : 0u;
    const uint32_t f = w < nw ? bmF[w] : 0u;
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
  return nsteps;
}

// rows r of a [rows x D] bf16 tile into 128-byte-swizzled 64-column boxes
__device__ __forceinline__ void store_row_swizzled(uint32_t tile, int box_bytes, int r,
                                                   const __nv_bfloat16* src, int D) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
  for (int i = 0; i < D / 8; ++i) {
    const uint4 u = src ? __ldg(s + i) : make_uint4(0u, 0u, 0u, 0u);
    st_shared_v4(tile + (i >> 3) * box_bytes + r * 128 + (((i & 7) ^ (r & 7)) << 4), u);
  }
}

// The walk of a CTA (run by warp 9): bitmaps A and B over the walked blocks
// (query pair: the kept key blocks of its two query blocks; key pair: the
// query blocks that kept either key block), bmF marks blocks without pad
// slots, then the step table.
__device__ __forceinline__ void bwd_walk(const Geo& g, const BwdIO& io, bool transposed, int pair,
                                         int bh, int b, int nw, uint32_t* bmA, uint32_t* bmB,
                                         uint32_t* bmF, uint16_t* steps, int* n_steps_sm,
                                         uint32_t bar_steps, int lane) {
  if (transposed) {
    const uint32_t* kt = io.kmask + (int64_t(bh) * g.nb) * nw;
    for (int w = lane; w < nw; w += 32) {
      bmA[w] = 2 * pair < g.nb ? __ldg(kt + int64_t(2 * pair) * nw + w) : 0u;
      bmB[w] = 2 * pair + 1 < g.nb ? __ldg(kt + int64_t(2 * pair + 1) * nw + w) : 0u;
    }
  } else {
    // a dense row keeps every block
    for (int w = lane; w < nw; w += 32) bmA[w] = bmB[w] = 0u;
    __syncwarp();
    for (int hf = 0; hf < 2; ++hf) {
      const int qb = 2 * pair + hf;
      if (qb >= g.nb) continue;
      uint32_t* bm = hf ? bmB : bmA;
      const int c = __ldg(io.cnt + int64_t(bh) * g.nb + qb);
      if (c < 0) {
        for (int w = lane; w < nw; w += 32) {
          const int rem = g.nb - 32 * w;
          bm[w] = rem >= 32 ? ~0u : ((1u << rem) - 1u);
        }
      } else {
        const int n = c < g.kcap ? c : g.kcap;
        const int32_t* src = io.idx + (int64_t(bh) * g.nb + qb) * g.kcap;
        for (int i = lane; i < n; i += 32) {
          const int v = __ldg(src + i);
          if (v >= 0 && v < g.nb) atomicOr(bm + (v >> 5), 1u << (v & 31));
        }
      }
    }
  }
  for (int w = lane; w < nw; w += 32) {
    uint32_t f = 0u;
    for (int i = 0; i < 32; ++i)
      if (32 * w + i < g.nb && __ldg(io.bfull + int64_t(b) * g.nb + 32 * w + i)) f |= 1u << i;
    bmF[w] = f;
  }
  __syncwarp();
  const int n = build_steps(bmA, bmB, bmF, nw, steps, lane);
  if (lane == 0) *n_steps_sm = n;
  __syncwarp();
  mbar_arrive(bar_steps);
}

// ============================================================================
// dQ: CTA = query pair, walk = union of the two key lists
// ============================================================================
template <int D>
__global__ void __launch_bounds__(320, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap mk, const __grid_constant__ CUtensorMap mv,
                       Geo g, const BwdIO io) {
  using C = BwdCfg<D>;
  constexpr int NS = C::NS;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* sm = smem_raw + (base - raw);
  const uint32_t sStg = base + C::OFF_STG;
  const BwdBars bb = bwd_bars<D>(base + C::OFF_BAR);
  uint32_t* bmA = reinterpret_cast<uint32_t*>(sm + C::OFF_BM);
  uint32_t* bmB = bmA + kMaxWords;
  uint32_t* bmF = bmA + 2 * kMaxWords;
  uint16_t* steps = reinterpret_cast<uint16_t*>(sm + C::OFF_STEPS);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + C::OFF_MISC + 4);
  int* n_steps_sm = reinterpret_cast<int*>(sm + C::OFF_MISC + 8);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x, bh = blockIdx.y, b = bh / g.h;
  auto stage_a = [&](int s) { return sStg + s * 2 * C::TILE64; };  // K
  auto stage_b = [&](int s) { return stage_a(s) + C::TILE64; };    // V

  if (threadIdx.x == 0) {
    bwd_init_bars<D>(bb);
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

  if (warp == 9) {
    bwd_walk(g, io, false, pair, bh, b, nw, bmA, bmB, bmF, steps, n_steps_sm, bb.steps, lane);
  } else if (warp == 8) {
    // ---- the issuer: copies and MMAs in step order
    if (lane == 0) {
      constexpr uint32_t idesc_sn = idesc_bf16_f32(128, 64, false);  // S, dP: B K-major
      constexpr uint32_t idesc_acc = idesc_bf16_f32(128, D, true);   // dQ: B N-major
      tma_prefetch_desc(&mk);
      tma_prefetch_desc(&mv);
      bool ok = mbar_wait(bb.steps, 0, abort_flag);
      const int n = ok ? *n_steps_sm : 0;
      auto load = [&](int j) {
        const int s = j % NS, t = int(steps[j] & kTileMask);
        mbar_arrive_expect_tx(bb.full + 8 * s, 2 * C::TILE64);
        for (int bx = 0; bx < C::KB; ++bx) {
          tma_load_3d(stage_a(s) + bx * C::BOX64, &mk, bb.full + 8 * s, 64 * bx, t * 64, bh);
          tma_load_3d(stage_b(s) + bx * C::BOX64, &mv, bb.full + 8 * s, 64 * bx, t * 64, bh);
        }
      };
      // step j's accumulation, dQ += dS_j K_j: A = group w's dS (tensor
      // memory, over its S columns), B = the K tile read N-major
      auto accumulate = [&](int j) -> bool {
        const int w = j & 1, s = j % NS;
        if (!mbar_wait(bb.x_ready + 8 * w, (j >> 1) & 1, abort_flag)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc_mma_ts(tmem + C::COL_DQ_ACC, tmem + C::COL_DQ_S + 128u * w + 8u * kk,
                    sdesc_sw128(stage_a(s) + kk * 2048, C::BOX64, 1024), idesc_acc,
                    (j > 0 || kk > 0) ? 1u : 0u);
        tc_commit(bb.x_free + 8 * w);
        tc_commit(bb.empty + 8 * s);
        return true;
      };
      int loaded = 0;  // steps whose copies have been issued
      if (n > 0) {
        load(0);
        loaded = 1;
      }
      ok = ok && mbar_wait(bb.own, 0, abort_flag);
      int j = 0;
      for (; ok && j < n; ++j) {
        const int w = j & 1, k = j >> 1, s = j % NS;
        // the next step's copies; its stage last held step j + 1 - NS,
        // whose accumulation was issued one iteration ago at the latest
        if (j + 1 < n) {
          if (j + 1 >= NS &&
              !mbar_wait(bb.empty + 8 * ((j + 1) % NS), ((j + 1 - NS) / NS) & 1, abort_flag)) {
            ok = false;
            break;
          }
          load(j + 1);
          loaded = j + 2;
        }
        // the accumulation of this group's previous step, then S_j = Q K_j^T
        // and dP_j = dO V_j^T into group w's columns once that accumulation
        // (which reads dS from them) has finished; A = Q or dO from tensor
        // memory, B = the K or V tile
        if (j >= 2 && !accumulate(j - 2)) {
          ok = false;
          break;
        }
        if (!mbar_wait(bb.full + 8 * s, (j / NS) & 1, abort_flag) ||
            (k > 0 && !mbar_wait(bb.x_free + 8 * w, (k - 1) & 1, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * C::BOX64 + (kk % 4) * 32;
          tc_mma_ts(tmem + C::COL_DQ_S + 128u * w, tmem + C::COL_DQ_Q + 8u * kk,
                    sdesc_sw128(stage_a(s) + off, 16, 1024), idesc_sn, kk > 0);
          tc_mma_ts(tmem + C::COL_DQ_S + 128u * w + 64u, tmem + C::COL_DQ_DO + 8u * kk,
                    sdesc_sw128(stage_b(s) + off, 16, 1024), idesc_sn, kk > 0);
        }
        tc_commit(bb.s_ready + 8 * w);
      }
      if (ok && n >= 2) ok = accumulate(n - 2);
      if (ok && n >= 1) ok = accumulate(n - 1);
      if (!ok) {
        report_timeout(abort_flag, io.status);
        // copies that may still be in flight: loaded steps from j on
        for (int jj = j; jj < loaded; ++jj)
          mbar_wait(bb.full + 8 * (jj % NS), (jj / NS) & 1, nullptr, 200000000ull);
      }
      tc_commit(bb.done);
      tc_commit(bb.drain);
      mbar_wait(bb.drain, 0, nullptr, 200000000ull);
    }
    __syncwarp();
  } else {
    // ---- row groups: group grp takes steps grp, grp + 2, ..; thread r of a
    // group owns row r of the pair = TMEM lane r
    const int grp = warp >> 2, quad = warp & 3;
    const int row = quad * 32 + lane, half = row >> 6, qb = 2 * pair + half;
    const uint32_t lane_base = uint32_t(quad * 32) << 16;
    const bool q_exists = qb < g.nb;
    const int64_t slot = int64_t(pair) * 128 + row;
    const bool row_valid =
        q_exists && ((__ldg(io.bmask + int64_t(b) * g.nb + qb) >> (row & 63)) & 1ull);
    const int64_t prow = int64_t(bh) * g.N + slot;
    // Q rows (group 0) and dO rows (group 1) into tensor memory, bf16 pairs
    // per column: the A operands of S and dP
    {
      const __nv_bfloat16* src = grp == 0 ? (q_exists ? io.q + prow * D : nullptr)
                                          : (row_valid ? io.dout + prow * D : nullptr);
      uint32_t rw[D / 2];
#pragma unroll
      for (int i = 0; i < D / 8; ++i) {
        const uint4 u = src ? __ldg(reinterpret_cast<const uint4*>(src) + i)
                            : make_uint4(0u, 0u, 0u, 0u);
        rw[4 * i] = u.x;
        rw[4 * i + 1] = u.y;
        rw[4 * i + 2] = u.z;
        rw[4 * i + 3] = u.w;
      }
      const uint32_t dst = tmem + (grp == 0 ? C::COL_DQ_Q : C::COL_DQ_DO) + lane_base;
      if constexpr (D == 128) {
        BSA_TMEM_ST64(dst, rw);
      } else {
        BSA_TMEM_ST32(dst, rw);
      }
      tc_fence_before();
    }
    mbar_arrive(bb.own);
    const float lse2 = row_valid ? __ldg(io.lse + prow) : INFINITY;
    const float dlt = row_valid ? __ldg(io.delta + prow) : 0.f;
    const float sl2 = g.scale * 1.4426950408889634f;
    const uint32_t tS = tmem + C::COL_DQ_S + 128u * grp + lane_base, tDP = tS + 64u;
    bool ok = __all_sync(0xffffffffu, mbar_wait(bb.steps, 0, abort_flag));
    const int n = ok ? *n_steps_sm : 0;
    int k = 0;
    for (int j = grp; ok && j < n; j += 2, ++k) {
      const uint32_t entry = steps[j];
      const int tile = int(entry & kTileMask);
      const uint32_t flags = entry >> kFlagShift;
      const bool member = row_valid && ((flags >> half) & 1u);
      ok = __all_sync(0xffffffffu, mbar_wait(bb.s_ready + 8 * grp, k & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      uint32_t sv[64], dp[64], pk[32];
      BSA_TMEM_LD64(tS, sv);
      BSA_TMEM_LD64(tDP, dp);
      if (member && (flags & 4u)) {
        // every key slot is a real token: two lanes per instruction
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          float x0, x1, t0, t1, d0, d1;
          fma_f32x2(x0, x1, __uint_as_float(sv[c]), __uint_as_float(sv[c + 1]), sl2, sl2, -lse2,
                    -lse2);
          const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
          add_f32x2(t0, t1, __uint_as_float(dp[c]), __uint_as_float(dp[c + 1]), -dlt, -dlt);
          fma_f32x2(d0, d1, p0, p1, t0, t1, 0.f, 0.f);
          pk[c / 2] = pack_bf16x2(d0, d1);
        }
      } else {
        const uint64_t vm = (flags & 4u) ? ~0ull : __ldg(io.bmask + int64_t(b) * g.nb + tile);
        const uint32_t lo = uint32_t(vm), hi = uint32_t(vm >> 32);
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          float d0 = 0.f, d1 = 0.f;
          if (member) {
            const float p0 =
                bit_of(lo, hi, c) ? ex2_approx(fmaf(__uint_as_float(sv[c]), sl2, -lse2)) : 0.f;
            const float p1 = bit_of(lo, hi, c + 1)
                                 ? ex2_approx(fmaf(__uint_as_float(sv[c + 1]), sl2, -lse2))
                                 : 0.f;
            d0 = p0 * (__uint_as_float(dp[c]) - dlt);
            d1 = p1 * (__uint_as_float(dp[c + 1]) - dlt);
          }
          pk[c / 2] = pack_bf16x2(d0, d1);
        }
      }
      // dS over this step's S (already read; the previous accumulation, which
      // read the previous dS there, finished before this step's S/dP)
      BSA_TMEM_ST32(tS, pk);
      tc_fence_before();
      mbar_arrive(bb.x_ready + 8 * grp);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bb.done, 0, abort_flag));
    if (!ok) {
      if (lane == 0) report_timeout(abort_flag, io.status);
    } else if (q_exists) {
      // group grp writes channels [grp * D/2, (grp + 1) * D/2)
      tc_fence_after();
      __nv_bfloat16* dst = io.dq + prow * D;
      const bool live = row_valid && n > 0;  // no steps: the accumulator was never written
#pragma unroll 1
      for (int ch = grp * (D / 64); ch < (grp + 1) * (D / 64); ++ch) {
        uint32_t a[32];
        BSA_TMEM_LD32(tmem + C::COL_DQ_ACC + 32u * ch + lane_base, a);
        uint32_t w16[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          w16[i] = pack_bf16x2(live ? __uint_as_float(a[2 * i]) * g.scale : 0.f,
                               live ? __uint_as_float(a[2 * i + 1]) * g.scale : 0.f);
        uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * ch);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          d4[i] = make_uint4(w16[4 * i], w16[4 * i + 1], w16[4 * i + 2], w16[4 * i + 3]);
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

// ============================================================================
// dK, dV: CTA = key pair, walk = union of the query blocks that kept them
// ============================================================================
template <int D>
__global__ void __launch_bounds__(320, 1)
    attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap mq,
                         const __grid_constant__ CUtensorMap mdo, Geo g, const BwdIO io) {
  using C = BwdCfg<D>;
  constexpr int NS = C::NS;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* sm = smem_raw + (base - raw);
  const uint32_t sK = base + C::OFF_OWN_A, sV = base + C::OFF_OWN_B, sStg = base + C::OFF_STG;
  const uint32_t sVec = base + C::OFF_VEC;
  const float* vec = reinterpret_cast<const float*>(sm + C::OFF_VEC);
  const BwdBars bb = bwd_bars<D>(base + C::OFF_BAR);
  uint32_t* bmA = reinterpret_cast<uint32_t*>(sm + C::OFF_BM);
  uint32_t* bmB = bmA + kMaxWords;
  uint32_t* bmF = bmA + 2 * kMaxWords;
  uint16_t* steps = reinterpret_cast<uint16_t*>(sm + C::OFF_STEPS);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + C::OFF_MISC + 4);
  int* n_steps_sm = reinterpret_cast<int*>(sm + C::OFF_MISC + 8);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x, bh = blockIdx.y, b = bh / g.h;
  auto stage_a = [&](int s) { return sStg + s * 2 * C::TILE64; };  // Q
  auto stage_b = [&](int s) { return stage_a(s) + C::TILE64; };    // dO

  if (threadIdx.x == 0) {
    bwd_init_bars<D>(bb);
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

  if (warp == 9) {
    bwd_walk(g, io, true, pair, bh, b, nw, bmA, bmB, bmF, steps, n_steps_sm, bb.steps, lane);
  } else if (warp == 8) {
    if (lane == 0) {
      constexpr uint32_t idesc_sn = idesc_bf16_f32(128, 64, false);
      constexpr uint32_t idesc_acc = idesc_bf16_f32(128, D, true);
      tma_prefetch_desc(&mq);
      tma_prefetch_desc(&mdo);
      bool ok = mbar_wait(bb.steps, 0, abort_flag);
      const int n = ok ? *n_steps_sm : 0;
      auto load = [&](int j) {
        const int s = j % NS, t = int(steps[j] & kTileMask);
        const int64_t r0 = int64_t(bh) * g.N + int64_t(t) * 64;
        mbar_arrive_expect_tx(bb.full + 8 * s, 2 * C::TILE64 + 2 * 256);
        for (int bx = 0; bx < C::KB; ++bx) {
          tma_load_3d(stage_a(s) + bx * C::BOX64, &mq, bb.full + 8 * s, 64 * bx, t * 64, bh);
          tma_load_3d(stage_b(s) + bx * C::BOX64, &mdo, bb.full + 8 * s, 64 * bx, t * 64, bh);
        }
        bulk_load(sVec + s * 512, io.lse + r0, 256, bb.full + 8 * s);
        bulk_load(sVec + s * 512 + 256, io.delta + r0, 256, bb.full + 8 * s);
      };
      // step j's accumulation: dV += P^T dO and dK += dS^T Q, A = group w's
      // P^T / dS^T (over its S / dP columns), B read N-major
      auto accumulate = [&](int j) -> bool {
        const int w = j & 1, s = j % NS;
        if (!mbar_wait(bb.x_ready + 8 * w, (j >> 1) & 1, abort_flag)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          tc_mma_ts(tmem + C::COL_DV, tmem + 128u * w + 8u * kk,
                    sdesc_sw128(stage_b(s) + kk * 2048, C::BOX64, 1024), idesc_acc,
                    (j > 0 || kk > 0) ? 1u : 0u);
          tc_mma_ts(tmem + C::COL_DK, tmem + 128u * w + 64u + 8u * kk,
                    sdesc_sw128(stage_a(s) + kk * 2048, C::BOX64, 1024), idesc_acc,
                    (j > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(bb.x_free + 8 * w);
        tc_commit(bb.empty + 8 * s);
        return true;
      };
      int loaded = 0;
      if (n > 0) {
        load(0);
        loaded = 1;
      }
      ok = ok && mbar_wait(bb.own, 0, abort_flag);
      int j = 0;
      for (; ok && j < n; ++j) {
        const int w = j & 1, k = j >> 1, s = j % NS;
        if (j + 1 < n) {
          if (j + 1 >= NS &&
              !mbar_wait(bb.empty + 8 * ((j + 1) % NS), ((j + 1 - NS) / NS) & 1, abort_flag)) {
            ok = false;
            break;
          }
          load(j + 1);
          loaded = j + 2;
        }
        // the accumulation of this group's previous step, then S^T_j = K Q_j^T
        // and dP^T_j = V dO_j^T into group w's columns once that accumulation
        // (which reads P^T and dS^T from those columns) has finished
        if (j >= 2 && !accumulate(j - 2)) {
          ok = false;
          break;
        }
        if (!mbar_wait(bb.full + 8 * s, (j / NS) & 1, abort_flag) ||
            (k > 0 && !mbar_wait(bb.x_free + 8 * w, (k - 1) & 1, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * C::BOX64 + (kk % 4) * 32;
          const uint32_t offo = (kk / 4) * C::BOX128 + (kk % 4) * 32;
          tc_mma_ss(tmem + 128u * w, sdesc_sw128(sK + offo, 16, 1024),
                    sdesc_sw128(stage_a(s) + off, 16, 1024), idesc_sn, kk > 0);
          tc_mma_ss(tmem + 128u * w + 64u, sdesc_sw128(sV + offo, 16, 1024),
                    sdesc_sw128(stage_b(s) + off, 16, 1024), idesc_sn, kk > 0);
        }
        tc_commit(bb.s_ready + 8 * w);
      }
      if (ok && n >= 2) ok = accumulate(n - 2);
      if (ok && n >= 1) ok = accumulate(n - 1);
      if (!ok) {
        report_timeout(abort_flag, io.status);
        for (int jj = j; jj < loaded; ++jj)
          mbar_wait(bb.full + 8 * (jj % NS), (jj / NS) & 1, nullptr, 200000000ull);
      }
      tc_commit(bb.done);
      tc_commit(bb.drain);
      mbar_wait(bb.drain, 0, nullptr, 200000000ull);
    }
    __syncwarp();
  } else {
    // ---- row groups: key row r of the pair = TMEM lane r
    const int grp = warp >> 2, quad = warp & 3;
    const int row = quad * 32 + lane, half = row >> 6, kb = 2 * pair + half;
    const uint32_t lane_base = uint32_t(quad * 32) << 16;
    const bool k_exists = kb < g.nb;
    const int64_t prow = int64_t(bh) * g.N + int64_t(pair) * 128 + row;
    const bool key_valid =
        k_exists && ((__ldg(io.bmask + int64_t(b) * g.nb + kb) >> (row & 63)) & 1ull);
    if (grp == 0)
      store_row_swizzled(sK, C::BOX128, row, k_exists ? io.k + prow * D : nullptr, D);
    else
      store_row_swizzled(sV, C::BOX128, row, k_exists ? io.v + prow * D : nullptr, D);
    fence_proxy_async_smem();
    mbar_arrive(bb.own);
    const float sl2 = g.scale * 1.4426950408889634f;
    const uint32_t tS = tmem + 128u * grp + lane_base, tDP = tS + 64u;
    bool ok = __all_sync(0xffffffffu, mbar_wait(bb.steps, 0, abort_flag));
    const int n = ok ? *n_steps_sm : 0;
    int k = 0;
    for (int j = grp; ok && j < n; j += 2, ++k) {
      const uint32_t entry = steps[j];
      const int tile = int(entry & kTileMask);
      const uint32_t flags = entry >> kFlagShift;
      const bool member = key_valid && ((flags >> half) & 1u);
      ok = __all_sync(0xffffffffu, mbar_wait(bb.s_ready + 8 * grp, k & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      uint32_t sv[64], dp[64];
      BSA_TMEM_LD64(tS, sv);
      BSA_TMEM_LD64(tDP, dp);
      // query slots of block `tile`: real tokens only (pad queries have no output)
      const uint64_t qm = (flags & 4u) ? ~0ull : __ldg(io.bmask + int64_t(b) * g.nb + tile);
      const uint32_t lo = uint32_t(qm), hi = uint32_t(qm >> 32);
      const float* lse = vec + (j % NS) * 128;
      const float* dlt = lse + 64;
      // P^T over S and dS^T over dP, 32 query columns (16 packed) at a time:
      // every column of S and dP is already in registers
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int c4 = 8 * h2; c4 < 8 * h2 + 8; ++c4) {
          // four columns' lse2 and D in one 16-byte load each
          const float4 l4 = reinterpret_cast<const float4*>(lse)[c4];
          const float4 t4 = reinterpret_cast<const float4*>(dlt)[c4];
          const float lv[4] = {l4.x, l4.y, l4.z, l4.w}, dv[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
          for (int u = 0; u < 4; u += 2) {
            const int c = 4 * c4 + u;
            float p0 = 0.f, p1 = 0.f, d0 = 0.f, d1 = 0.f;
            if (member && (flags & 4u)) {
              // every query slot is a real token: two lanes per instruction
              float x0, x1, t0, t1;
              fma_f32x2(x0, x1, __uint_as_float(sv[c]), __uint_as_float(sv[c + 1]), sl2, sl2,
                        -lv[u], -lv[u + 1]);
              p0 = ex2_approx(x0);
              p1 = ex2_approx(x1);
              add_f32x2(t0, t1, __uint_as_float(dp[c]), __uint_as_float(dp[c + 1]), -dv[u],
                        -dv[u + 1]);
              fma_f32x2(d0, d1, p0, p1, t0, t1, 0.f, 0.f);
            } else if (member) {
              if (bit_of(lo, hi, c)) {
                p0 = ex2_approx(fmaf(__uint_as_float(sv[c]), sl2, -lv[u]));
                d0 = p0 * (__uint_as_float(dp[c]) - dv[u]);
              }
              if (bit_of(lo, hi, c + 1)) {
                p1 = ex2_approx(fmaf(__uint_as_float(sv[c + 1]), sl2, -lv[u + 1]));
                d1 = p1 * (__uint_as_float(dp[c + 1]) - dv[u + 1]);
              }
            }
            pk[(c - 32 * h2) / 2] = pack_bf16x2(p0, p1);
            dk[(c - 32 * h2) / 2] = pack_bf16x2(d0, d1);
          }
        }
        BSA_TMEM_ST16(tS + 16u * h2, pk);
        BSA_TMEM_ST16(tDP + 16u * h2, dk);
      }
      tc_fence_before();
      mbar_arrive(bb.x_ready + 8 * grp);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bb.done, 0, abort_flag));
    if (!ok) {
      if (lane == 0) report_timeout(abort_flag, io.status);
    } else if (k_exists) {
      // group 0 writes dV, group 1 dK (scaled)
      tc_fence_after();
      __nv_bfloat16* dst = (grp ? io.dk : io.dv) + prow * D;
      const float f = grp ? g.scale : 1.f;
      // a key block no query kept has no steps and zero gradients (its
      // accumulators were never written)
      const bool live = key_valid && n > 0;
#pragma unroll 1
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t a[32];
        BSA_TMEM_LD32(tmem + (grp ? C::COL_DK : C::COL_DV) + 32u * ch + lane_base, a);
        uint32_t w16[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          w16[i] = pack_bf16x2(live ? __uint_as_float(a[2 * i]) * f : 0.f,
                               live ? __uint_as_float(a[2 * i + 1]) * f : 0.f);
        uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * ch);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          d4[i] = make_uint4(w16[4 * i], w16[4 * i + 1], w16[4 * i + 2], w16[4 * i + 3]);
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

// ============================================================================
// D = rowsum(dO * O) and the transposed (key block -> query blocks) bitmaps
// ============================================================================
__global__ void __launch_bounds__(256) bwd_delta_kernel(Geo g, const __nv_bfloat16* __restrict__ o,
                                                        const __nv_bfloat16* __restrict__ dout,
                                                        float* __restrict__ delta) {
  // 8 threads per row, each 16 bytes at a time
  const int64_t rows = int64_t(g.B) * g.h * g.N;
  const int64_t r = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 3;
  const int sub = threadIdx.x & 7;
  float acc = 0.f;
  if (r < rows) {
    const uint4* po = reinterpret_cast<const uint4*>(o + r * g.d);
    const uint4* pd = reinterpret_cast<const uint4*>(dout + r * g.d);
    for (int i = sub; i < g.d / 8; i += 8) {
      const uint4 a = __ldg(po + i), c = __ldg(pd + i);
      const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
      const __nv_bfloat162* c2 = reinterpret_cast<const __nv_bfloat162*>(&c);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 x = __bfloat1622float2(a2[k]), y = __bfloat1622float2(c2[k]);
        acc = fmaf(x.x, y.x, acc);
        acc = fmaf(x.y, y.y, acc);
      }
    }
  }
#pragma unroll
  for (int off = 4; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (r < rows && sub == 0) delta[r] = acc;
}

// kmask[bh][key block j] bit i: query block i keeps j (a dense row keeps all)
__global__ void __launch_bounds__(256) bwd_transpose_kernel(Geo g, const int32_t* __restrict__ idx,
                                                            const int32_t* __restrict__ cnt,
                                                            uint32_t* __restrict__ kmask) {
  const int i = blockIdx.x, bh = blockIdx.y;
  const int nw = (g.nb + 31) >> 5;
  uint32_t* km = kmask + int64_t(bh) * g.nb * nw;
  const uint32_t bit = 1u << (i & 31);
  const int c = cnt[int64_t(bh) * g.nb + i];
  if (c < 0) {
    for (int j = threadIdx.x; j < g.nb; j += blockDim.x) atomicOr(km + int64_t(j) * nw + (i >> 5), bit);
  } else {
    const int n = c < g.kcap ? c : g.kcap;
    const int32_t* src = idx + (int64_t(bh) * g.nb + i) * g.kcap;
    for (int e = threadIdx.x; e < n; e += blockDim.x) {
      const int j = src[e];
      if (j >= 0 && j < g.nb) atomicOr(km + int64_t(j) * nw + (i >> 5), bit);
    }
  }
}

template <int D>
cudaError_t launch_bwd_t(const Geo& g, const CUtensorMap* maps, const BwdIO& io, cudaStream_t st) {
  using C = BwdCfg<D>;
  const int nw = (g.nb + 31) >> 5;
  cudaError_t e = cudaMemsetAsync(io.kmask, 0, sizeof(uint32_t) * size_t(g.B) * g.h * g.nb * nw, st);
  if (e != cudaSuccess) return e;
  bwd_transpose_kernel<<<dim3(g.nb, g.B * g.h), 256, 0, st>>>(g, io.idx, io.cnt, io.kmask);
  const int64_t rows = int64_t(g.B) * g.h * g.N;
  bwd_delta_kernel<<<unsigned((rows * 8 + 255) / 256), 256, 0, st>>>(g, io.o, io.dout, io.delta);
  e = cudaFuncSetAttribute(attn_bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::SMEM);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(attn_bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::SMEM);
  if (e != cudaSuccess) return e;
  const dim3 grid((g.nb + 1) / 2, g.B * g.h);
  attn_bwd_dq_kernel<D><<<grid, C::kThreads, C::SMEM, st>>>(maps[0], maps[1], g, io);
  attn_bwd_dkdv_kernel<D><<<grid, C::kThreads, C::SMEM, st>>>(maps[2], maps[3], g, io);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention_bwd(const Geo& g, const CUtensorMap* maps, const BwdIO& io,
                                 cudaStream_t st) {
  return g.d == 128 ? launch_bwd_t<128>(g, maps, io, st) : launch_bwd_t<64>(g, maps, io, st);
}

}  // namespace bsa
