// Block-sparse attention forward on sm_100a: TMA-fed tcgen05 tiles with the
// accumulators in tensor memory, walking a per-query-block list of kept key
// blocks so that only kept 64x64 tiles are ever loaded or multiplied
// (Sparse VideoGen on TPU, aibase.it, section "이론적 sparsity와 물리적
// sparsity의 차이": skipping empty tiles is where the speed comes from).
//
// CTA = two adjacent query blocks (128 query rows = the full tcgen05 M=128
// datapath; M=64 would leave half of it idle).  The two blocks' sorted key
// lists are merged on the fly; each merged step loads one 64-token key
// block (K and V, 16 KB each at head_dim 128) and computes
//     S = Q K^T      (M=128, N=64,  K=head_dim)  -> TMEM, double buffered
//     O += P V       (M=128, N=head_dim, K=64)   -> TMEM accumulator
// Rows of a block that did not keep the step's key block get P = 0.
//
// Warp roles (192 threads):
//   warps 0-3  softmax + epilogue; thread r owns query row r = TMEM lane r
//   warp 4     TMA producer: Q once, then K/V per step into a ring
//   warp 5     TMEM allocator and single-thread tcgen05.mma issuer
// Softmax is the exact online softmax in the exp2 domain with a lazily
// updated running max: the O rescale is only applied when the row max grows
// by more than 2^8, which keeps every probability below 256 (still exact
// after the final division by the running sum).
//
// Every wait is bounded (2 s); a timeout sets the caller's status word to
// BSA_ERR_TIMEOUT, drains in-flight copies and MMAs and frees tensor memory.
#include <climits>

#include "bsa_internal.cuh"

namespace bsa {
namespace {

template <int D>
struct Cfg {
  static constexpr int kThreads = 192;
  static constexpr int BM = 128, BN = 64;
  static constexpr int STAGES = (D == 128) ? 4 : 6;
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int P_BYTES = BM * BN * 2;
  static constexpr int Q_BOX = BM * 128;  // bytes of one 64-column Q box
  static constexpr int KV_BOX = BN * 128;
  static constexpr uint32_t TMEM_COLS = 256;  // S0 [0,64) S1 [64,128) O [128,128+D)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * KV_BYTES;
  static constexpr int OFF_P = OFF_V + STAGES * KV_BYTES;
  static constexpr int OFF_BAR = OFF_P + P_BYTES;
  static constexpr int N_BARS = 2 * STAGES + 6;
  static constexpr int OFF_INFO = OFF_BAR + 8 * N_BARS;
  static constexpr int OFF_MISC = OFF_INFO + 16 * STAGES;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;  // + slack for 1024-B alignment
};

struct StepInfo {
  int32_t tile;    // key block, or -1 = no more steps
  uint32_t flags;  // bit 0: first query block keeps it; bit 1: second one
  uint64_t vmask;  // valid-slot mask of the key block
};

// Iterator over the kept key blocks of one query block.
struct ListIt {
  const int32_t* p;
  int n, pos, dense_n;
  __device__ int peek() const {
    if (dense_n) return pos < dense_n ? pos : INT_MAX;
    return pos < n ? __ldg(p + pos) : INT_MAX;
  }
};

__device__ __forceinline__ void report_timeout(volatile int* abort_flag, int32_t* status) {
  *abort_flag = 1;
  atomicCAS(status, 0, int32_t(BSA_ERR_TIMEOUT));
}

template <int D, bool DENSE>
__global__ void __launch_bounds__(192, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                    const __grid_constant__ CUtensorMap mv, Geo g,
                    const uint64_t* __restrict__ bmask, const int32_t* __restrict__ idx,
                    const int32_t* __restrict__ cnt, __nv_bfloat16* __restrict__ out,
                    int32_t* __restrict__ status) {
  using C = Cfg<D>;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* sm = smem_raw + (base - raw);
  const uint32_t sQ = base + C::OFF_Q, sK = base + C::OFF_K, sV = base + C::OFF_V,
                 sP = base + C::OFF_P, bar0 = base + C::OFF_BAR;
  // barrier ids
  const uint32_t bar_q = bar0 + 8 * (2 * C::STAGES);
  const uint32_t bar_s = bar_q + 8;      // two: S buffer 0 / 1 ready
  const uint32_t bar_p = bar_q + 24;     // P written + O corrected (128 arrivals)
  const uint32_t bar_o = bar_q + 32;     // PV finished
  const uint32_t bar_drain = bar_q + 40; // final MMA drain
  StepInfo* info = reinterpret_cast<StepInfo*>(sm + C::OFF_INFO);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x, bh = blockIdx.y, b = bh / g.h;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(bar0 + 8 * s, 1);
      mbar_init(bar0 + 8 * (C::STAGES + s), 1);
    }
    mbar_init(bar_q, 1);
    mbar_init(bar_s, 1);
    mbar_init(bar_s + 8, 1);
    mbar_init(bar_p, 128);
    mbar_init(bar_o, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t tS = tmem, tO = tmem + 128;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&mq);
      tma_prefetch_desc(&mk);
      tma_prefetch_desc(&mv);
      mbar_arrive_expect_tx(bar_q, C::Q_BYTES);
      for (int bx = 0; bx < D / 64; ++bx)
        tma_load_3d(sQ + bx * C::Q_BOX, &mq, bar_q, bx * 64, pair * 128, bh);
      ListIt it[2];
      for (int hf = 0; hf < 2; ++hf) {
        const int qb = 2 * pair + hf;
        it[hf] = {nullptr, 0, 0, 0};
        if (qb < g.nb) {
          const int c = DENSE ? -1 : __ldg(cnt + int64_t(bh) * g.nb + qb);
          if (c < 0)
            it[hf].dense_n = g.nb;
          else {
            it[hf].p = idx + (int64_t(bh) * g.nb + qb) * g.kcap;
            it[hf].n = c;
          }
        }
      }
      int j = 0;
      bool ok = true;
      for (;; ++j) {
        const int s = j % C::STAGES;
        if (j >= C::STAGES &&
            !mbar_wait(bar0 + 8 * (C::STAGES + s), ((j / C::STAGES) - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        const int ta = it[0].peek(), tb = it[1].peek();
        const int t = ta < tb ? ta : tb;
        if (t == INT_MAX) {
          info[s].tile = -1;
          mbar_arrive(bar0 + 8 * s);
          break;
        }
        uint32_t flags = 0;
        if (ta == t) { flags |= 1u; ++it[0].pos; }
        if (tb == t) { flags |= 2u; ++it[1].pos; }
        info[s].tile = t;
        info[s].flags = flags;
        info[s].vmask = __ldg(bmask + int64_t(b) * g.nb + t);
        const uint32_t full = bar0 + 8 * s;
        mbar_arrive_expect_tx(full, 2 * C::KV_BYTES);
        for (int bx = 0; bx < D / 64; ++bx) {
          tma_load_3d(sK + s * C::KV_BYTES + bx * C::KV_BOX, &mk, full, bx * 64, t * 64, bh);
          tma_load_3d(sV + s * C::KV_BYTES + bx * C::KV_BOX, &mv, full, bx * 64, t * 64, bh);
        }
      }
      if (!ok) {
        report_timeout(abort_flag, status);
        // let the copies already in flight land before the CTA goes away
        for (int jj = j - 1; jj >= 0 && jj >= j - C::STAGES; --jj)
          mbar_wait(bar0 + 8 * (jj % C::STAGES), (jj / C::STAGES) & 1, nullptr, 200000000ull);
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 64, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, true);
      bool ok = mbar_wait(bar_q, 0, abort_flag);
      for (int j = 0; ok; ++j) {
        const int s = j % C::STAGES;
        if (!mbar_wait(bar0 + 8 * s, (j / C::STAGES) & 1, abort_flag)) {
          ok = false;
          break;
        }
        const int tile = *reinterpret_cast<volatile int32_t*>(&info[s].tile);
        if (tile >= 0) {
          tc_fence_after();
          const uint32_t dS = tS + uint32_t(j & 1) * 64u;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t a = sdesc_sw128(sQ + (kk / 4) * C::Q_BOX + (kk % 4) * 32, 16, 1024);
            const uint64_t bd =
                sdesc_sw128(sK + s * C::KV_BYTES + (kk / 4) * C::KV_BOX + (kk % 4) * 32, 16, 1024);
            tc_mma_ss(dS, a, bd, idesc_qk, kk > 0 ? 1u : 0u);
          }
          tc_commit(bar_s + 8 * (j & 1));
        }
        if (j > 0) {
          const int jp = j - 1, sp = jp % C::STAGES;
          if (!mbar_wait(bar_p, jp & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t a = sdesc_sw128(sP + kk * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(sV + sp * C::KV_BYTES + kk * 2048, C::KV_BOX, 1024);
            tc_mma_ss(tO, a, bd, idesc_pv, (jp > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(bar_o);
          tc_commit(bar0 + 8 * (C::STAGES + sp));
        }
        if (tile < 0) break;
      }
      if (!ok) report_timeout(abort_flag, status);
      // every MMA this thread issued has completed once bar_drain flips
      tc_commit(bar_drain);
      mbar_wait(bar_drain, 0, nullptr, 200000000ull);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int row = warp * 32 + lane;
    const int half = warp >> 1;
    const int qb = 2 * pair + half;
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    const bool q_exists = qb < g.nb;
    const bool row_valid =
        q_exists && ((__ldg(bmask + int64_t(b) * g.nb + qb) >> (row & 63)) & 1ull);
    const float sl2 = g.scale * 1.4426950408889634f;
    float m_used = -INFINITY, l_sum = 0.f;
    bool ok = true;
    int j = 0;
    for (;; ++j) {
      const int s = j % C::STAGES;
      ok = __all_sync(0xffffffffu, mbar_wait(bar0 + 8 * s, (j / C::STAGES) & 1, abort_flag));
      if (!ok) break;
      const int tile = *reinterpret_cast<volatile int32_t*>(&info[s].tile);
      if (tile < 0) break;
      const uint32_t flags = *reinterpret_cast<volatile uint32_t*>(&info[s].flags);
      const uint64_t vm = *reinterpret_cast<volatile uint64_t*>(&info[s].vmask);
      const bool member = (flags >> half) & 1u;
      ok = __all_sync(0xffffffffu, mbar_wait(bar_s + 8 * (j & 1), (j >> 1) & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      uint32_t pk[32];
      float factor = 1.f;
      bool rescale = false;
      if (member) {
        uint32_t r[64];
        const uint32_t ts = tS + uint32_t(j & 1) * 64u + lane_base;
        BSA_TMEM_LD32(ts, r);
        BSA_TMEM_LD32(ts + 32, (r + 32));
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if ((vm >> c) & 1ull) mx = fmaxf(mx, __uint_as_float(r[c]));
        const float mxs = mx * sl2;
        if (mxs > m_used + 8.f) {
          if (m_used != -INFINITY) {
            factor = ex2_approx(m_used - mxs);
            rescale = true;
          }
          m_used = mxs;
        }
        float sum = 0.f;
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          const float p0 = ((vm >> c) & 1ull) ? ex2_approx(fmaf(__uint_as_float(r[c]), sl2, -m_used)) : 0.f;
          const float p1 =
              ((vm >> (c + 1)) & 1ull) ? ex2_approx(fmaf(__uint_as_float(r[c + 1]), sl2, -m_used)) : 0.f;
          sum += p0 + p1;
          pk[c / 2] = pack_bf16x2(p0, p1);
        }
        l_sum = l_sum * factor + sum;
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = 0u;
      }
      // P buffer and O are free once the previous PV has finished
      if (j > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar_o, (j - 1) & 1, abort_flag));
        if (!ok) break;
      }
      if (__any_sync(0xffffffffu, rescale)) {
        tc_fence_after();
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t o[32];
          const uint32_t ta = tO + uint32_t(ch * 32) + lane_base;
          BSA_TMEM_LD32(ta, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * factor);
          BSA_TMEM_ST32(ta, o);
        }
      }
      const uint32_t prow = sP + uint32_t(row) * 128u;
#pragma unroll
      for (int c16 = 0; c16 < 8; ++c16) {
        const uint32_t addr = prow + (uint32_t(c16 ^ (row & 7)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pk[4 * c16]),
                     "r"(pk[4 * c16 + 1]), "r"(pk[4 * c16 + 2]), "r"(pk[4 * c16 + 3])
                     : "memory");
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar_p);
    }
    // ---------------------------------------------------------- epilogue
    if (ok && j > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar_o, (j - 1) & 1, abort_flag));
    if (!ok) {
      if (lane == 0) report_timeout(abort_flag, status);
    } else if (q_exists) {
      tc_fence_after();
      const float inv = (row_valid && l_sum > 0.f) ? 1.f / l_sum : 0.f;
      __nv_bfloat16* orow = out + (int64_t(bh) * g.N + int64_t(qb) * 64 + (row & 63)) * D;
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t o[32];
        BSA_TMEM_LD32(tO + uint32_t(ch * 32) + lane_base, o);
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          w[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
        uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int D, bool DENSE>
cudaError_t launch_t(const Geo& g, LayoutPtrs lp, const CUtensorMap* maps, const int32_t* idx,
                     const int32_t* cnt, __nv_bfloat16* o, int32_t* status, cudaStream_t st) {
  using C = Cfg<D>;
  auto kern = attn_fwd_kernel<D, DENSE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid((g.nb + 1) / 2, g.B * g.h);
  kern<<<grid, C::kThreads, C::SMEM, st>>>(maps[0], maps[1], maps[2], g, lp.bmask, idx, cnt, o,
                                           status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const Geo& g, LayoutPtrs lp, const CUtensorMap* maps,
                             const int32_t* idx, const int32_t* cnt, __nv_bfloat16* o,
                             int32_t* dev_status, bool dense, cudaStream_t st) {
  if (g.d == 128)
    return dense ? launch_t<128, true>(g, lp, maps, idx, cnt, o, dev_status, st)
                 : launch_t<128, false>(g, lp, maps, idx, cnt, o, dev_status, st);
  return dense ? launch_t<64, true>(g, lp, maps, idx, cnt, o, dev_status, st)
               : launch_t<64, false>(g, lp, maps, idx, cnt, o, dev_status, st);
}

}  // namespace bsa
