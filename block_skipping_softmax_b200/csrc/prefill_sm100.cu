// Skip Softmax prefill attention for sm_100a (B200).
//
// Method: "Accelerating Long-Context Inference with Skip Softmax in NVIDIA
// TensorRT-LLM" (Key Points; Detailed Analysis).  Key tiles are visited in
// ascending order; a tile is skipped -- no exponentials, no P*V MMA, no V
// load -- iff every row of the row block has tile max < running max - tau.
// Otherwise the usual online-softmax update runs (block-wise attention that
// never materialises the N x N score matrix, as the TurboAttention talk page
// describes FlashAttention in its Technical Deep Dive).
//
// One CTA owns one row block (Br query rows of one head) and runs four roles:
//   warp 0      TMA producer for Q (once) and the K tiles (ring of KS stages)
//   warp 1      TMEM allocator and the single MMA-issuing thread:
//                 S_j = Q K_j^T  (SS tcgen05.mma, fp32 in TMEM, two buffers)
//                 O  += P_j V_j  (TS tcgen05.mma, P read from TMEM)
//   warp 2      TMA producer for the V tiles; under a finite tau it loads V_j
//               only after the skip decision for tile j keeps it
//   warps 4-7   softmax: thread r owns query row r (TMEM lane r); it loads S_j,
//               forms the tile max, votes on the skip, and for kept tiles
//               writes P_j = exp2(S_j - m) (bf16) back into TMEM over S_j,
//               rescales O when the reference max moves, and stores O / l.
// Every wait is bounded; a wait that gives up records ATTN_ERR_TIMEOUT in the
// status word and the CTA unwinds without trapping.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.cuh"
#include "ptx.cuh"

namespace bss {

namespace {

constexpr int kThreads = 256;
constexpr int kMmaM = 128;         // tcgen05 tile height; Br = 64 uses rows 0..63
constexpr int kDecRing = 4;        // skip decisions in flight between roles
constexpr float kRescaleLog2 = 8.0f;  // O/l are rescaled only when the max grows by > 2^8

template <int D, int BC>
struct PrefillCfg {
  static constexpr int kPanels = D / 64;                  // 128-byte swizzle panels per row
  static constexpr int kQBytes = kMmaM * D * 2;
  static constexpr int kKVBytes = BC * D * 2;
  static constexpr int kQPanel = kMmaM * 128;
  static constexpr int kKVPanel = BC * 128;
  static constexpr int kStages = (D == 128 && BC == 128) ? 2 : 3;
  static constexpr int kTmemCols = (D + 2 * BC <= 256) ? 256 : 512;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + kStages * kKVBytes;
  static constexpr int kOffBar = kOffV + kStages * kKVBytes;
  // barriers: q_full, k_full[S], k_empty[S], v_full[S], v_empty[S], s_full[2],
  // p_full[2], pv_done, o_final, dec_full[kDecRing]
  static constexpr int kNumBars = 1 + 4 * kStages + 2 + 2 + 1 + 1 + kDecRing;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  // + misc + alignment slack; a CTA that takes all 512 TMEM columns also asks
  // for enough shared memory that no second CTA shares its SM (a second one
  // would only stall in tcgen05.alloc)
  static constexpr int kSmemUsed = kOffMisc + 128 + 1024;
  static constexpr int kSmemBytes =
      (kTmemCols == 512 && kSmemUsed < 120 * 1024) ? 120 * 1024 : kSmemUsed;
};

struct Misc {
  uint32_t tmem_base;
  int abort;
  int dec[kDecRing];
  int vote[2][4];
};

__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ void give_up(Misc* misc, int* status, int where) {
  reinterpret_cast<volatile int*>(&misc->abort)[0] = 1;
  atomicCAS(status, 0, ATTN_DEVICE_TIMEOUT_BASE + where);
}

}  // namespace

template <int D, int BR, int BC, bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, __nv_bfloat16* __restrict__ O,
                   uint8_t* __restrict__ skip_mask, int* __restrict__ status, int B, int Hq,
                   int Hkv, int N, float scale_log2, float tau_log2, int tau_is_inf,
                   unsigned long long wait_limit_ns) {
  using C = PrefillCfg<D, BC>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + C::kOffQ;
  const uint32_t sK = sbase + C::kOffK;
  const uint32_t sV = sbase + C::kOffV;
  const uint32_t bar0 = sbase + C::kOffBar;
  const uint32_t b_q_full = bar0;
  auto b_k_full = [&](int s) { return bar0 + 8u * (1 + s); };
  auto b_k_empty = [&](int s) { return bar0 + 8u * (1 + C::kStages + s); };
  auto b_v_full = [&](int s) { return bar0 + 8u * (1 + 2 * C::kStages + s); };
  auto b_v_empty = [&](int s) { return bar0 + 8u * (1 + 3 * C::kStages + s); };
  auto b_s_full = [&](int i) { return bar0 + 8u * (1 + 4 * C::kStages + i); };
  auto b_p_full = [&](int i) { return bar0 + 8u * (3 + 4 * C::kStages + i); };
  const uint32_t b_pv_done = bar0 + 8u * (5 + 4 * C::kStages);
  const uint32_t b_o_final = bar0 + 8u * (6 + 4 * C::kStages);
  auto b_dec_full = [&](int i) { return bar0 + 8u * (7 + 4 * C::kStages + i); };
  Misc* misc = reinterpret_cast<Misc*>(smem + C::kOffMisc);
  volatile int* abort_flag = &misc->abort;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work item: (row block, batch*head).  Causal: the longest row blocks
  // run first, heads fastest (the g heads of a KV group share K/V in L2).
  // Non-causal: row blocks fastest, so the CTAs that read one head's K/V run
  // together and the re-reads hit L2.
  const int n_rb = (N + BR - 1) / BR;
  const int BH = B * Hq;
  const int bh = CAUSAL ? static_cast<int>(blockIdx.x % BH) : static_cast<int>(blockIdx.x / n_rb);
  const int rb = CAUSAL ? (n_rb - 1 - static_cast<int>(blockIdx.x / BH))
                        : static_cast<int>(blockIdx.x % n_rb);
  const int b = bh / Hq;
  const int h = bh % Hq;
  const int g = Hq / Hkv;
  const int bkv = b * Hkv + h / g;
  const int n_tiles = (N + BC - 1) / BC;
  const int last_row = min(N, (rb + 1) * BR) - 1;
  const int T = CAUSAL ? (last_row / BC + 1) : n_tiles;  // tiles visited

  if (threadIdx.x == 0) {
    mbar_init(b_q_full, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(b_k_full(s), 1);
      mbar_init(b_k_empty(s), 1);
      mbar_init(b_v_full(s), 1);
      mbar_init(b_v_empty(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(b_s_full(i), 1);
      mbar_init(b_p_full(i), 4);
    }
    mbar_init(b_pv_done, 1);
    mbar_init(b_o_final, 1);
    for (int i = 0; i < kDecRing; ++i) mbar_init(b_dec_full(i), 1);
    misc->abort = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&misc->tmem_base), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc->tmem_base;
  const uint32_t tO = tmem;                                   // columns [0, D)
  auto tS = [&](int i) { return tmem + D + i * BC; };          // two S/P buffers

  if (warp == 0) {
    // ------------------------------------------------ producer: Q and K tiles
    if (lane == 0) {
      const int bq = b * Hq + h;
      mbar_arrive_expect_tx(b_q_full, C::kQBytes);
      for (int p = 0; p < C::kPanels; ++p)
        tma_load_3d(sQ + p * C::kQPanel, &tmQ, b_q_full, p * 64, rb * BR, bq);
      int issued = 0;
      for (int j = 0; j < T; ++j) {
        const int s = j % C::kStages;
        if (j >= C::kStages &&
            !mbar_wait(b_k_empty(s), ((j / C::kStages) - 1) & 1, abort_flag, wait_limit_ns)) {
          give_up(misc, status, 1);
          break;
        }
        mbar_arrive_expect_tx(b_k_full(s), C::kKVBytes);
        for (int p = 0; p < C::kPanels; ++p)
          tma_load_3d(sK + s * C::kKVBytes + p * C::kKVPanel, &tmK, b_k_full(s), p * 64, j * BC,
                      bkv);
        ++issued;
      }
      // never leave while a copy into this CTA's shared memory is in flight
      mbar_drain(b_q_full, 0, wait_limit_ns);
      for (int t = max(0, issued - C::kStages); t < issued; ++t)
        mbar_drain(b_k_full(t % C::kStages), (t / C::kStages) & 1, wait_limit_ns);
    }
  } else if (warp == 2) {
    // ------------------------------------------------ producer: V tiles of kept tiles
    if (lane == 0) {
      int kept = 0;
      for (int j = 0; j < T; ++j) {
        int keep = 1;
        if (!tau_is_inf) {
          const int di = j % kDecRing;
          if (!mbar_wait(b_dec_full(di), (j / kDecRing) & 1, abort_flag, wait_limit_ns)) {
            give_up(misc, status, 2);
            break;
          }
          keep = reinterpret_cast<volatile int*>(misc->dec)[di];
        }
        if (!keep) continue;
        const int s = kept % C::kStages;
        if (kept >= C::kStages &&
            !mbar_wait(b_v_empty(s), ((kept / C::kStages) - 1) & 1, abort_flag, wait_limit_ns)) {
          give_up(misc, status, 3);
          break;
        }
        mbar_arrive_expect_tx(b_v_full(s), C::kKVBytes);
        for (int p = 0; p < C::kPanels; ++p)
          tma_load_3d(sV + s * C::kKVBytes + p * C::kKVPanel, &tmV, b_v_full(s), p * 64, j * BC,
                      bkv);
        ++kept;
      }
      for (int t = max(0, kept - C::kStages); t < kept; ++t)
        mbar_drain(b_v_full(t % C::kStages), (t / C::kStages) & 1, wait_limit_ns);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer (one thread)
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(kMmaM, BC, false, false);
      constexpr uint32_t idPV = idesc_bf16_f32(kMmaM, D, false, true);
      bool ok = mbar_wait(b_q_full, 0, abort_flag, wait_limit_ns);
      if (!ok) give_up(misc, status, 4);
      int kept = 0;
      for (int j = 0; ok && j <= T; ++j) {
        if (j < T) {
          const int s = j % C::kStages;
          if (!mbar_wait(b_k_full(s), (j / C::kStages) & 1, abort_flag, wait_limit_ns)) {
            give_up(misc, status, 5);
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk & 3) * 32;  // 16 bf16 = 32 B inside a 128 B row
            const uint64_t da = sw128_desc(sQ + (kk >> 2) * C::kQPanel + off, 16, 1024);
            const uint64_t db =
                sw128_desc(sK + s * C::kKVBytes + (kk >> 2) * C::kKVPanel + off, 16, 1024);
            mma_ss(tS(j & 1), da, db, idS, kk > 0 ? 1u : 0u);
          }
          mma_commit(b_s_full(j & 1));
          mma_commit(b_k_empty(s));
        }
        if (j >= 1) {
          const int i = j - 1;
          if (!mbar_wait(b_p_full(i & 1), (i >> 1) & 1, abort_flag, wait_limit_ns)) {
            give_up(misc, status, 6);
            break;
          }
          tc_fence_after();
          const int keep = reinterpret_cast<volatile int*>(misc->dec)[i % kDecRing];
          if (keep) {
            const int s = kept % C::kStages;
            if (!mbar_wait(b_v_full(s), (kept / C::kStages) & 1, abort_flag, wait_limit_ns)) {
              give_up(misc, status, 7);
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < BC / 16; ++kk) {
              const uint64_t db =
                  sw128_desc(sV + s * C::kKVBytes + kk * 16 * 128, C::kKVPanel, 1024);
              mma_ts(tO, tS(i & 1) + kk * 8, db, idPV, (kept > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(b_v_empty(s));
            mma_commit(b_pv_done);
            ++kept;
          }
        }
      }
      mma_commit(b_o_final);
      // all issued MMAs must finish before TMEM is released
      mbar_drain(b_o_final, 0, wait_limit_ns);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------ softmax warpgroup
    const int sw = warp - 4;
    const int row = sw * 32 + lane;
    const int q_idx = rb * BR + row;
    const bool row_valid = (row < BR) && (q_idx < N);
    const uint32_t lane_off = static_cast<uint32_t>(sw * 32) << 16;
    const float NEG_INF = -__int_as_float(0x7f800000);
    float m_exact = NEG_INF;  // exact running row max (log2 units) -- drives the skip test
    float m_ref = NEG_INF;    // reference max of the exponentials (lags by < 2^8)
    float l_sum = 0.f;
    int kept = 0;
    bool ok = true;
    bool failed = false;  // this warp gave up on a wait; acted on at the next vote
    const size_t mask_base = skip_mask ? ((static_cast<size_t>(bh) * n_rb + rb) * n_tiles) : 0;

    for (int j = 0; j < T; ++j) {
      const int sb = j & 1;
      // warp-uniform result: the TMEM loads below are warp-collective
      bool waited = !failed && __all_sync(0xffffffffu, mbar_wait(b_s_full(sb), (j >> 1) & 1,
                                                                  abort_flag, wait_limit_ns));
      float x[BC];
      float mt = NEG_INF;
      if (waited) {
        tc_fence_after();
        uint32_t r[BC];
#pragma unroll
        for (int c0 = 0; c0 < BC; c0 += 32)
          tmem_ld32(tS(sb) + lane_off + c0, *reinterpret_cast<uint32_t(*)[32]>(&r[c0]));
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < BC; ++c) x[c] = __uint_as_float(r[c]) * scale_log2;
        const int key0 = j * BC;
        const bool need_mask = (key0 + BC > N) || (CAUSAL && key0 + BC - 1 > rb * BR);
        if (!row_valid) {
#pragma unroll
          for (int c = 0; c < BC; ++c) x[c] = NEG_INF;
        } else if (need_mask) {
#pragma unroll
          for (int c = 0; c < BC; ++c) {
            const int key = key0 + c;
            if (key >= N || (CAUSAL && key > q_idx)) x[c] = NEG_INF;
          }
        }
#pragma unroll
        for (int c = 0; c < BC; ++c) mt = fmaxf(mt, x[c]);
      }
      // ---- the block-skip test: skip iff every row has mt < m - tau
      bool skip = false;
      if (!tau_is_inf) {
        const bool pass =
            !row_valid || (m_exact != NEG_INF && (mt == NEG_INF || mt < m_exact - tau_log2));
        const unsigned all_pass = __all_sync(0xffffffffu, pass);
        const unsigned all_waited = __all_sync(0xffffffffu, waited);
        if (lane == 0)
          reinterpret_cast<volatile int*>(misc->vote[sb])[sw] =
              (all_pass ? 1 : 0) | (all_waited ? 0 : 2);
        named_bar_sync(1, 128);
        int v = 1, bad = 0;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const int vw = reinterpret_cast<volatile int*>(misc->vote[sb])[w];
          v &= vw & 1;
          bad |= vw & 2;
        }
        skip = v != 0;
        if (bad) waited = false;
      }
      if (!waited) {
        give_up(misc, status, 8);
        ok = false;
        break;
      }
      m_exact = fmaxf(m_exact, mt);
      if (row == 0) {
        reinterpret_cast<volatile int*>(misc->dec)[j % kDecRing] = skip ? 0 : 1;
        if (skip_mask) skip_mask[mask_base + j] = skip ? 1 : 0;
        mbar_arrive(b_dec_full(j % kDecRing));
      }
      if (skip) {
        __syncwarp();
        if (lane == 0) mbar_arrive(b_p_full(sb));
        continue;
      }
      // ---- kept tile: online softmax update with a lazily moved reference max
      const float m_cand = fmaxf(m_ref, mt);
      const bool moved = row_valid && (m_cand > m_ref + kRescaleLog2);
      float alpha = 1.f;
      if (moved) {
        alpha = ex2(m_ref - m_cand);  // m_ref = -inf on the first tile gives 0
        m_ref = m_cand;
      }
      // P = 2^(x - m_ref) as bf16 pairs, written over this row's S columns
      // (64 scores -> 32 packed columns per store).  The row sum adds the
      // bf16-rounded values that the P*V MMA multiplies, so numerator and
      // denominator see the same weights and the rounding of a dominant
      // weight cancels in O / l.
      float rs = 0.f;
#pragma unroll
      for (int c0 = 0; c0 < BC; c0 += 64) {
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          float p0 = ex2(x[c0 + 2 * c] - m_ref);
          float p1 = ex2(x[c0 + 2 * c + 1] - m_ref);
          if (!row_valid) p0 = p1 = 0.f;
          const uint32_t w = pack_bf16x2(p0, p1);
          rs += __uint_as_float(w << 16) + __uint_as_float(w & 0xffff0000u);
          pk[c] = w;
        }
        tmem_st32(tS(sb) + lane_off + c0 / 2, pk);
      }
      l_sum = l_sum * alpha + rs;
      const bool need_o = moved && kept > 0;
      if (__any_sync(0xffffffffu, need_o)) {
        // O is read-modify-written: the last issued P*V must have finished
        if (!__all_sync(0xffffffffu,
                        mbar_wait(b_pv_done, (kept - 1) & 1, abort_flag, wait_limit_ns))) {
          // leave O alone; the other softmax warps learn of it at the next
          // vote (breaking here could strand them at the named barrier)
          give_up(misc, status, 9);
          failed = true;
        } else {
          tc_fence_after();
          const float a = need_o ? alpha : 1.f;
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t r[32];
            tmem_ld32(tO + lane_off + c0, r);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) r[c] = __float_as_uint(__uint_as_float(r[c]) * a);
            tmem_st32(tO + lane_off + c0, r);
          }
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0 && !failed) mbar_arrive(b_p_full(sb));
      ++kept;
      if (failed && tau_is_inf) {  // no votes without a finite tau: stop here
        ok = false;
        break;
      }
    }
    if (failed) ok = false;

    // ---- epilogue: O / l -> bf16 -> global
    if (skip_mask)
      for (int j = T + row; j < n_tiles; j += 128) skip_mask[mask_base + j] = 2;
    if (__all_sync(0xffffffffu, ok && mbar_wait(b_o_final, 0, abort_flag, wait_limit_ns))) {
      tc_fence_after();
      const float inv_l = row_valid ? 1.f / l_sum : 0.f;
      __nv_bfloat16* orow = O + (static_cast<size_t>(bh) * N + (row_valid ? q_idx : 0)) * D;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(tO + lane_off + c0, r);
        tmem_wait_ld();
        if (row_valid) {
          uint32_t w[16];
#pragma unroll
          for (int c = 0; c < 16; ++c)
            w[c] = pack_bf16x2(__uint_as_float(r[2 * c]) * inv_l,
                               __uint_as_float(r[2 * c + 1]) * inv_l);
          uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
        }
      }
    } else if (ok) {
      give_up(misc, status, 10);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// --------------------------------------------------------------------- host
namespace {

PFN_cuTensorMapEncodeTiled_v12000 get_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// [BH, rows, D] bf16, d fastest; box = 64 columns x box_rows rows, 128 B swizzle
bool make_map(CUtensorMap* m, const void* base, int BH, int rows, int D, int box_rows) {
  auto enc = get_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2,
                           static_cast<cuuint64_t>(rows) * D * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, int BR, int BC, bool CAUSAL>
int launch(const PrefillLaunch& a) {
  using C = PrefillCfg<D, BC>;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, a.Q, a.B * a.Hq, a.N, D, kMmaM) ||
      !make_map(&mk, a.K, a.B * a.Hkv, a.N, D, BC) ||
      !make_map(&mv, a.V, a.B * a.Hkv, a.N, D, BC))
    return ATTN_ERR_CUDA;
  auto kern = prefill_kernel<D, BR, BC, CAUSAL>;
  static uint64_t attr_done = 0;  // one bit per device ordinal
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  if (dev < 64 && !(attr_done >> dev & 1)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
        cudaSuccess)
      return ATTN_ERR_CUDA;
    attr_done |= uint64_t(1) << dev;
  }
  const long long n_rb = (a.N + BR - 1) / BR;
  const long long grid = n_rb * a.B * a.Hq;
  if (grid > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  kern<<<static_cast<unsigned>(grid), kThreads, C::kSmemBytes, a.stream>>>(
      mq, mk, mv, static_cast<__nv_bfloat16*>(a.O), a.skip_mask, a.status, a.B, a.Hq, a.Hkv, a.N,
      a.scale_log2, a.tau_log2, a.tau_is_inf, a.wait_limit_ns);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <int D, int BR, int BC>
int launch_c(const PrefillLaunch& a) {
  return a.causal ? launch<D, BR, BC, true>(a) : launch<D, BR, BC, false>(a);
}

template <int D>
int launch_d(const PrefillLaunch& a) {
  if (a.Br == 64 && a.Bc == 64) return launch_c<D, 64, 64>(a);
  if (a.Br == 128 && a.Bc == 64) return launch_c<D, 128, 64>(a);
  if (a.Br == 128 && a.Bc == 128) return launch_c<D, 128, 128>(a);
  return ATTN_ERR_INVALID_ARG;
}

}  // namespace

int launch_prefill(const PrefillLaunch& a) {
  if (a.d == 64) return launch_d<64>(a);
  if (a.d == 128) return launch_d<128>(a);
  return ATTN_ERR_INVALID_ARG;
}

}  // namespace bss
