// Skip Softmax prefill for sm_100a, d = 128: one 128-row block per work
// item, the two softmax warpgroups splitting each key tile by columns;
// persistent over work items.
//
// Method: "Accelerating Long-Context Inference with Skip Softmax in NVIDIA
// TensorRT-LLM" (Key Points; Detailed Analysis): key tiles are visited in
// ascending order, and key tile t of a row block is skipped -- no
// exponentials, no P*V product, no V load -- iff every row of the row block
// has its tile maximum strictly below its running maximum minus tau.
//
// Why this layout.  With d = 128, the 512 TMEM columns hold the O
// accumulator of one 128-row block (128 columns) and three S buffers of 128
// keys.  The S MMAs of the next two key tiles therefore run while the softmax
// works on the current one, so nothing forces the chain S_j -> softmax ->
// P*V_j -> S_{j+1} of a layout that keeps two row blocks (two O
// accumulators) in TMEM.  Each 128-key S tile is shared by both softmax
// warpgroups: warpgroup h takes key columns [64h, 64h + 64) of every row.
// The two halves' row maxima are exchanged through shared memory once per
// tile, so both halves compute P against the same reference maximum and one
// P*V product (P read from the two TMEM column ranges) accumulates one O.
//
// Skip granularity BC: 128 (one decision per S tile) or 64 (the two halves
// of S tile j are the rule's key tiles 2j and 2j + 1; half B is tested
// against the running maximum that already includes half A's tile maximum,
// as the ascending visiting order requires).
//
// Roles (384 threads, one CTA per SM):
//   warp 0: TMA of Q (two slots, the next item's Q loads during this one)
//           and of the K ring;
//   warp 1: TMEM allocation and the MMA-issuing thread;
//   warp 2: TMA of the V ring, gated by the skip decisions;
//   warp 3: idle;
//   warpgroup 1 (warps 4-7): softmax of key columns 0-63 of each S tile;
//   warpgroup 2 (warps 8-11): key columns 64-127.
// TMEM: O at columns [0, 128), S buffer b at [128 + 128b, 256 + 128b); the
// bf16 P of half h is written over the first 32 columns of that half.
// Shared memory: Q slots 2 x 32 KB, K ring 3 x 32 KB, V ring 2 x 32 KB, then
// barriers and the exchange buffers; O is staged in the item's finished Q
// slot and written by two TMA stores (one 64-column panel per warpgroup).
//
// Completion signalling.  The issuer commits once per S tile of the
// prologue and once per key tile of the main loop, into a ring of mbarriers
// indexed by a running commit count:
//   S of S tile i ready         commit #(base + i)
//   P*V of S tile j finished    commit #(base + min(SB, T) + j)
// (one thread issues every MMA, and a commit covers all its earlier MMAs).
// Every wait is bounded; a role that gives up records a status code and
// the CTA unwinds, leaving no copy or MMA in flight and freeing TMEM.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "exp2_poly.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace bss {

namespace {

constexpr int kThreads = 384;
constexpr int kRegs = 168;           // registers per thread at launch (checked on the host)
constexpr int kRows = 128;           // query rows per work item
constexpr int kD = 128;              // head dimension
constexpr int kST = 128;             // keys per S tile
constexpr int kSB = 3;               // S buffers in TMEM
constexpr int kQS = 2, kKS = 3, kVS = 2;
constexpr int kCR = 16;              // commit ring
constexpr int kDR = 4;               // decision ring
constexpr int kTile = kRows * kD * 2;  // 32 KB: one Q, K, V or O tile in bf16
constexpr int kPanel = kRows * 128;    // 16 KB: 64 columns x 128 rows
constexpr int kHalfPanel = 64 * 128;   // 8 KB: 64 columns x 64 rows
constexpr float kRescale = 8.0f;       // lazy rescale threshold (log2 units)
constexpr int kProducerRegs = 72;
constexpr int kSoftmaxRegs = (kThreads * kRegs - 128 * kProducerRegs) / 256 / 8 * 8;
static_assert(128 * kProducerRegs + 256 * kSoftmaxRegs <= kThreads * kRegs, "register split");
static_assert(kD + kSB * kST <= 512, "TMEM budget");
static_assert(kKS + kSB + 1 < kCR && kVS + kSB + 1 < kCR, "commit ring too small");

// shared-memory layout
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kQS * kTile;
constexpr int kOffV = kOffK + kKS * kTile;
constexpr int kOffMisc = kOffV + kVS * kTile;
// barriers: k_full[KS], v_full[VS], commit ring[CR], p_full[SB], q_full[QS],
// q_empty[QS], mma_done
constexpr int kBK = 0, kBV = kBK + kKS, kBC = kBV + kVS, kBP = kBC + kCR, kBQF = kBP + kSB,
              kBQE = kBQF + kQS, kBM = kBQE + kQS, kNumBars = kBM + 1;
constexpr int kOffTmem = kOffMisc + kNumBars * 8;
constexpr int kOffAbort = kOffTmem + 4;
constexpr int kOffVote = kOffAbort + 4;                 // int [kDR][2][4]
constexpr int kOffLeave = kOffVote + kDR * 2 * 4 * 4;   // int [2][8]
constexpr int kOffXm = kOffMisc + 1024;                 // float [2][2][128]
constexpr int kSmemBytes = kOffXm + 2 * 2 * kRows * 4;
static_assert(kOffLeave + 2 * 8 * 4 <= kOffXm, "misc layout");
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");


__device__ __forceinline__ void give_up(volatile int* abort_flag, int* status, int where) {
  *abort_flag = 1;
  atomicCAS(status, 0, ATTN_DEVICE_TIMEOUT_BASE + 64 + where);
}

// One work item: query head bh (batch-major), row block rb; T S tiles are
// visited, and T64 key tiles of 64 (the rule's tiles when BC = 64).
struct Item {
  int bh, rb, T, T64;
};

template <bool CAUSAL>
__device__ __forceinline__ Item make_item(long long idx, int BH, int n_rb, int N, int g,
                                          bool group_major) {
  Item it;
  if (CAUSAL && group_major) {
    // KV-head groups one after another (longest row blocks first inside a
    // group, heads fastest): the CTAs in flight share one group's K/V, which
    // then stays in L2 however long the sequence
    const long long per_group = static_cast<long long>(g) * n_rb;
    const int grp = static_cast<int>(idx / per_group);
    const int r = static_cast<int>(idx % per_group);
    it.rb = n_rb - 1 - r / g;
    it.bh = grp * g + r % g;
  } else if (CAUSAL) {  // longest row blocks first, heads fastest
    it.rb = n_rb - 1 - static_cast<int>(idx / BH);
    it.bh = static_cast<int>(idx % BH);
  } else {  // row blocks fastest: the CTAs reading one head's K/V run together
    it.rb = static_cast<int>(idx % n_rb);
    it.bh = static_cast<int>(idx / n_rb);
  }
  const int last = min(N, (it.rb + 1) * kRows) - 1;  // last row of the block
  if (CAUSAL) {
    it.T = last / kST + 1;
    it.T64 = last / 64 + 1;
  } else {
    it.T = (N + kST - 1) / kST;
    it.T64 = (N + 63) / 64;
  }
  return it;
}

// Ring-slot releases waiting to be checked: the commit number that covers
// the slot's last reader, and (V ring) the running tile number of that
// reader.  Fixed positions keep the entries in registers.
struct Pending3 {
  int c[3], g[3], n;
  __device__ __forceinline__ void init() { n = 0; }
  __device__ __forceinline__ void push(int cc, int gg) {
    if (n == 0) { c[0] = cc; g[0] = gg; }
    else if (n == 1) { c[1] = cc; g[1] = gg; }
    else { c[2] = cc; g[2] = gg; }
    ++n;
  }
  __device__ __forceinline__ void pop() {
    c[0] = c[1]; g[0] = g[1];
    c[1] = c[2]; g[1] = g[2];
    --n;
  }
};

}  // namespace

// POLY: which of the 16 column pairs of each 32-column chunk take the
// polynomial exp2 on the FMA pipes instead of MUFU (bit c = pair c; 0 = all
// on MUFU).  SKIP: tau is finite, so the kernel takes the skip test; with
// tau = inf it holds no trace of it (the test's branches alone cost the
// softmax loop about 6 % in scheduling).
template <int BC, bool CAUSAL, uint32_t POLY, bool SKIP>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_split_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                         uint8_t* __restrict__ skip_mask, int* __restrict__ status, int B, int Hq,
                         int Hkv, int N, float scale_log2, float tau_log2,
                         unsigned long long wait_limit_ns) {
  static_assert(BC == 64 || BC == 128, "skip granularity");
  constexpr bool kHalves = BC == 64;  // two rule tiles per S tile
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  // the swizzled TMA boxes and MMA descriptors need 1024-byte alignment; the
  // layout uses the whole 227 KB and keeps no slack to realign, so a base
  // that is not aligned is reported (site 99) before anything is started
  if (sbase & 1023u) {
    if (threadIdx.x == 0) atomicCAS(status, 0, ATTN_DEVICE_TIMEOUT_BASE + 64 + 35);
    return;
  }
  const uint32_t sQ = sbase + kOffQ, sK = sbase + kOffK, sV = sbase + kOffV;
  const uint32_t bar0 = sbase + kOffMisc;
  auto b_k_full = [&](int s) { return bar0 + 8u * (kBK + s); };
  auto b_v_full = [&](int s) { return bar0 + 8u * (kBV + s); };
  auto b_cm = [&](int i) { return bar0 + 8u * (kBC + (i % kCR)); };
  auto b_p_full = [&](int b) { return bar0 + 8u * (kBP + b); };
  auto b_q_full = [&](int s) { return bar0 + 8u * (kBQF + s); };
  auto b_q_empty = [&](int s) { return bar0 + 8u * (kBQE + s); };
  const uint32_t b_mma_done = bar0 + 8u * kBM;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffAbort);
  // vote[i][h][w]: (decision number << 2) | 2 if warp w of warpgroup h gave
  // up | 1 if every row of that warp passes the skip test of warpgroup h's
  // tile, for the decision in ring slot i (one decision number per S tile)
  volatile int* vote = reinterpret_cast<volatile int*>(smem + kOffVote);
  auto vote_at = [&](int i, int h, int w) { return vote + (i * 2 + h) * 4 + w; };
  volatile int* leave = reinterpret_cast<volatile int*>(smem + kOffLeave);
  volatile float* xm = reinterpret_cast<volatile float*>(smem + kOffXm);  // [2][2][128]
  auto decided_keep = [&](int h, int i) -> int {
    return ((*vote_at(i, h, 0) & *vote_at(i, h, 1) & *vote_at(i, h, 2) & *vote_at(i, h, 3)) & 1) ? 0 : 1;
  };
  auto wait_cm = [&](int i) { return mbar_wait(b_cm(i), (i / kCR) & 1, abort_flag, wait_limit_ns); };
  // all four votes of warpgroup h for decision number dnum (ring slot i) are
  // in; false if the wait gave up (the abort flag, or the time limit)
  auto votes_in = [&](int h, int i, int dnum) -> bool {
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t n = 0;; ++n) {
      bool all = true;
#pragma unroll
      for (int w = 0; w < 4; ++w) all = all && ((*vote_at(i, h, w) >> 2) == dnum);
      if (all) return true;
      if ((n & 15u) == 15u && (*abort_flag || globaltimer_ns() - t0 > wait_limit_ns)) return false;
      __nanosleep(96);
    }
  };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_rb = (N + kRows - 1) / kRows;
  const int BH = B * Hq;
  const int g = Hq / Hkv;
  const long long n_items = static_cast<long long>(BH) * n_rb;
  // Causal layers whose KV-head groups hold many items per CTA (long
  // sequences) go group by group, so the K/V that the CTAs in flight read
  // fits in L2 (the 128K-token 70B layer: 537 MB of K/V, 67 MB per group);
  // with few items per group, a round would mix long and short items and
  // unbalance the CTAs, so heads stay fastest there.
  const bool group_major = CAUSAL && static_cast<long long>(g) * n_rb >= 8LL * gridDim.x;
  // The k-th work item of this CTA: rounds of gridDim.x items; causal items
  // (longest first) go out in a "snake", CTAs ascending in even rounds and
  // descending in odd ones, which evens out the work per CTA.
  auto item_idx = [&](long long k) -> long long {
    const long long G = gridDim.x;
    return k * G + ((CAUSAL && (k & 1)) ? G - 1 - blockIdx.x : blockIdx.x);
  };
  const int n_dec = kHalves ? (N + 63) / 64 : (N + kST - 1) / kST;  // mask row length

  if (threadIdx.x == 0) {
    for (int s = 0; s < kKS; ++s) mbar_init(b_k_full(s), 1);
    for (int s = 0; s < kVS; ++s) mbar_init(b_v_full(s), 1);
    for (int i = 0; i < kCR; ++i) mbar_init(b_cm(i), 1);
    for (int b = 0; b < kSB; ++b) mbar_init(b_p_full(b), 8);  // one arrival per softmax warp
    for (int s = 0; s < kQS; ++s) {
      mbar_init(b_q_full(s), 1);
      mbar_init(b_q_empty(s), 2);  // one per warpgroup's O store
    }
    mbar_init(b_mma_done, 1);
    for (int i = 0; i < kDR * 2 * 4; ++i) vote[i] = -1;  // no decision number matches
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(sbase + kOffTmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + kOffTmem);
  const uint32_t tO = tmem;
  auto tS = [&](int b) { return tmem + kD + b * kST; };

  if (warp < 4) {
    reg_dec<kProducerRegs>();
    if (warp == 0 && lane == 0) {
      // ------------------------------------------------------ Q and K producer
      int kload = 0, items = 0, base = 0;
      Pending3 pend;
      pend.init();
      bool alive = true;
      for (long long k = 0, idx = item_idx(0); alive && idx < n_items; idx = item_idx(++k)) {
        const Item it = make_item<CAUSAL>(idx, BH, n_rb, N, g, group_major);
        const int bkv = (it.bh / Hq) * Hkv + (it.bh % Hq) / g;
        const int qs = items % kQS;
        if (items >= kQS &&
            !mbar_wait(b_q_empty(qs), ((items / kQS) - 1) & 1, abort_flag, wait_limit_ns)) {
          give_up(abort_flag, status, 1);
          break;
        }
        mbar_arrive_expect_tx(b_q_full(qs), kTile);
        for (int p = 0; p < 2; ++p)
          tma_load_3d(sQ + qs * kTile + p * kPanel, &tmQ, b_q_full(qs), p * 64, it.rb * kRows, it.bh);
        ++items;
        for (int j = 0; j < it.T; ++j) {
          if (pend.n == kKS) {  // the slot's previous tile: its S MMA must have run
            if (!wait_cm(pend.c[0])) {
              give_up(abort_flag, status, 2);
              alive = false;
              break;
            }
            pend.pop();
          }
          const int s = kload % kKS;
          mbar_arrive_expect_tx(b_k_full(s), kTile);
          for (int p = 0; p < 2; ++p)
            tma_load_3d(sK + s * kTile + p * kPanel, &tmK, b_k_full(s), p * 64, j * kST, bkv);
          pend.push(base + j, 0);  // S of S tile j is commit #(base + j)
          ++kload;
        }
        base += min(kSB, it.T) + it.T;
      }
      // never leave with a copy in flight
      for (int i = max(0, items - kQS); i < items; ++i)
        mbar_drain(b_q_full(i % kQS), (i / kQS) & 1, wait_limit_ns);
      for (int t = max(0, kload - kKS); t < kload; ++t)
        mbar_drain(b_k_full(t % kKS), (t / kKS) & 1, wait_limit_ns);
    } else if (warp == 2 && lane == 0) {
      // ------------------------------------------------------ V producer
      int vload = 0, dl = 0, base = 0, gbase = 0;
      Pending3 pend;
      pend.init();
      bool alive = true;
      for (long long k = 0, idx = item_idx(0); alive && idx < n_items; idx = item_idx(++k)) {
        const Item it = make_item<CAUSAL>(idx, BH, n_rb, N, g, group_major);
        const int bkv = (it.bh / Hq) * Hkv + (it.bh % Hq) / g;
        const int pro = min(kSB, it.T);
        for (int j = 0; alive && j < it.T; ++j) {
          bool keepA = true;
          bool keepB = !kHalves || 2 * j + 1 < it.T64;
          if (SKIP) {
            // every decision is consumed in order; the V of S tile j (or of
            // each kept half) is loaded once some part of it is kept
            // the softmax warps publish their votes without a barrier
            // arrival (an arrival is a long-latency step on their path from S
            // to P); this thread polls the vote words of decision dl, with a
            // bounded wait
            const int di = dl % kDR;
            if (!votes_in(0, di, dl) || !votes_in(1, di, dl)) {
              give_up(abort_flag, status, 3);
              alive = false;
              break;
            }
            ++dl;
            keepA = kHalves ? decided_keep(0, di) : (decided_keep(0, di) | decided_keep(1, di));
            keepB = kHalves ? (keepB && decided_keep(1, di)) : keepA;
          }
          if (!keepA && !keepB) continue;
          if (pend.n == kVS) {
            // The slot's previous tile: its P*V MMAs must have run.  Once a
            // decision on S tile j has been read, S_j has completed, and with
            // it every MMA issued before it, which includes every P*V of S
            // tiles j - SB and earlier (items are SB apart in the running
            // tile number).  Those commits are not waited for: after a run of
            // skipped tiles their ring slot may have been reused.
            const bool known_done = SKIP && pend.g[0] + kSB < gbase + j;
            if (!known_done && !wait_cm(pend.c[0])) {
              give_up(abort_flag, status, 4);
              alive = false;
              break;
            }
            pend.pop();
          }
          const int s = vload % kVS;
          const uint32_t dst = sV + s * kTile;
          if (!kHalves) {
            mbar_arrive_expect_tx(b_v_full(s), kTile);
            for (int p = 0; p < 2; ++p)
              tma_load_3d(dst + p * kPanel, &tmV, b_v_full(s), p * 64, j * kST, bkv);
          } else {
            mbar_arrive_expect_tx(b_v_full(s), (keepA ? kTile / 2 : 0) + (keepB ? kTile / 2 : 0));
            for (int hh = 0; hh < 2; ++hh)
              if (hh == 0 ? keepA : keepB)
                for (int p = 0; p < 2; ++p)
                  tma_load_3d(dst + p * kPanel + hh * kHalfPanel, &tmV, b_v_full(s), p * 64,
                              j * kST + hh * 64, bkv);
          }
          pend.push(base + pro + j, gbase + j);  // P*V of S tile j is commit #(base + pro + j)
          ++vload;
        }
        base += pro + it.T;
        gbase += it.T + kSB;
      }
      for (int t = max(0, vload - kVS); t < vload; ++t)
        mbar_drain(b_v_full(t % kVS), (t / kVS) & 1, wait_limit_ns);
    } else if (warp == 1 && lane == 0) {
      // ------------------------------------------------------ MMA issuer
      constexpr uint32_t idS = idesc_bf16_f32(kRows, kST, false, false);
      constexpr uint32_t idPV = idesc_bf16_f32(kRows, kD, false, true);
      // descriptors differ only in their start-address field (bits 0-13, in
      // 16-byte units): each MMA adds a compile-time offset to a 32-bit base
      constexpr uint32_t kHi = sw128_desc_hi(1024);
      const uint32_t dK0 = sw128_desc_lo(sK, 16);
      const uint32_t dV0 = sw128_desc_lo(sV, kPanel);
      int kuse = 0, vuse = 0, items = 0, pc = 0, sq = 0, cmc = 0, dc = 0;
      bool alive = true;
      auto wait_k = [&]() -> bool {
        if (!mbar_wait(b_k_full(kuse % kKS), (kuse / kKS) & 1, abort_flag, wait_limit_ns)) {
          give_up(abort_flag, status, 6);
          return false;
        }
        tc_fence_after();
        return true;
      };
      auto issue_S = [&](uint32_t dQ) {  // S tile into buffer sq % SB from K slot kuse % KS
        const uint32_t b0 = dK0 + (kuse % kKS) * (kTile >> 4);
        const uint32_t d = tS(sq % kSB);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {  // 32 bytes of the reduction each
          const uint32_t off = ((kk >> 2) * kPanel + (kk & 3) * 32) >> 4;
          mma_ss(d, desc_join(dQ + off, kHi), desc_join(b0 + off, kHi), idS, kk > 0 ? 1u : 0u);
        }
        ++sq;
        ++kuse;
      };
      auto commit = [&]() {
        mma_commit(b_cm(cmc));
        ++cmc;
      };
      for (long long k = 0, idx = item_idx(0); alive && idx < n_items; idx = item_idx(++k)) {
        const Item it = make_item<CAUSAL>(idx, BH, n_rb, N, g, group_major);
        const int qs = items % kQS;
        const uint32_t dQ = sw128_desc_lo(sQ + qs * kTile, 16);
        if (!mbar_wait(b_q_full(qs), (items / kQS) & 1, abort_flag, wait_limit_ns)) {
          give_up(abort_flag, status, 5);
          break;
        }
        ++items;
        const int pro = min(kSB, it.T);
        for (int jj = 0; jj < pro; ++jj) {  // S of the first SB tiles, one commit each
          if (!wait_k()) {
            alive = false;
            break;
          }
          issue_S(dQ);
          commit();
        }
        if (!alive) break;
        bool started = false;  // the item's first P*V MMA overwrites O
        for (int j = 0; j < it.T; ++j) {
          const int pb = pc % kSB;
          if (!mbar_wait(b_p_full(pb), (pc / kSB) & 1, abort_flag, wait_limit_ns)) {
            give_up(abort_flag, status, 7);
            alive = false;
            break;
          }
          ++pc;
          tc_fence_after();
          // every softmax warp wrote its vote before arriving on p_full
          bool keepA = true;
          bool keepB = !kHalves || 2 * j + 1 < it.T64;
          if (SKIP) {
            const int di = dc % kDR;
            keepA = kHalves ? decided_keep(0, di) : (decided_keep(0, di) | decided_keep(1, di));
            keepB = kHalves ? (keepB && decided_keep(1, di)) : keepA;
          }
          ++dc;
          if (keepA || keepB) {
            if (!mbar_wait(b_v_full(vuse % kVS), (vuse / kVS) & 1, abort_flag, wait_limit_ns)) {
              give_up(abort_flag, status, 8);
              alive = false;
              break;
            }
            tc_fence_after();
            const uint32_t vb = dV0 + (vuse % kVS) * (kTile >> 4);
#pragma unroll
            for (int kk = 0; kk < kST / 16; ++kk) {
              // keys [16kk, 16kk + 16): P of half kk / 4 at columns 64 * (kk / 4) + 8 * (kk % 4)
              if (kk < 4 ? !keepA : !keepB) continue;
              mma_ts(tO, tS(pb) + (kk >> 2) * 64 + (kk & 3) * 8,
                     desc_join(vb + ((kk * 16 * 128) >> 4), kHi), idPV, started ? 1u : 0u);
              started = true;
            }
            ++vuse;
          }
          if (j + kSB < it.T) {  // S of tile j + SB reuses the buffer P_j just left
            if (!wait_k()) {
              alive = false;
              break;
            }
            issue_S(dQ);
          }
          commit();  // #(base + pro + j): P*V_j and S_{j+SB}
        }
      }
      // all issued MMAs must finish before TMEM is released
      mma_commit(b_mma_done);
      mbar_drain(b_mma_done, 0, wait_limit_ns);
    }
  } else {
    reg_inc<kSoftmaxRegs>();
    // -------------------------------------------------------- softmax warpgroups
    const int h = (warp - 4) >> 2;  // key-column half of every S tile
    const int sw = warp & 3;        // TMEM sub-partition of this warp
    const int row = sw * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(sw * 32) << 16;
    const float NEG_INF = -__int_as_float(0x7f800000);
    const float sl2 = scale_log2;
    const float2 sc2 = make_float2(sl2, sl2);
    int sc = 0, xc = 0, dcount = 0, base = 0, items = 0, leaves = 0;
    // thread 0 of each warpgroup: the Q slot its last O store reads
    int pend_slot = -1;
    auto release_pending = [&]() {
      if (pend_slot >= 0) {
        bulk_wait_read_all();
        mbar_arrive(b_q_empty(pend_slot));
        pend_slot = -1;
      }
    };
    // exchange of one float per row with the other warpgroup's thread of the
    // same row: both warpgroups call it the same number of times
    auto exchange = [&](float mine) -> float {
      volatile float* slot = xm + (xc & 1) * 2 * kRows;
      slot[h * kRows + row] = mine;
      named_bar(1, 256);
      const float other = slot[(1 - h) * kRows + row];
      ++xc;
      return other;
    };
    bool ok = true, failed = false;
    for (long long k = 0, idx = item_idx(0); ok && idx < n_items; idx = item_idx(++k)) {
      const Item it = make_item<CAUSAL>(idx, BH, n_rb, N, g, group_major);
      const int qs = items % kQS;
      ++items;
      const int pro = min(kSB, it.T);
      const int q_idx = it.rb * kRows + row;
      const bool row_valid = q_idx < N;
      const size_t mask_base = skip_mask ? (static_cast<size_t>(it.bh) * n_rb + it.rb) * n_dec : 0;
      float m_exact = NEG_INF, m_ref = NEG_INF, l_h = 0.f;
      for (int j = 0; j < it.T; ++j) {
        const int sb = sc % kSB;
        ++sc;
        bool waited = !failed && __all_sync(0xffffffffu, wait_cm(base + j));
        uint32_t u[64];
        float mh = NEG_INF;  // this half's tile maximum, log2 units
        if (waited) {
          tc_fence_after();
          tmem_ld_row<64>(tS(sb) + h * 64 + lane_off, u);
          tmem_wait_ld();
          // last visible column of this row in this half (-1: none)
          const int key0 = j * kST + h * 64;
          int lim = min(63, N - 1 - key0);
          if (CAUSAL) lim = min(lim, q_idx - key0);
          if (!row_valid) lim = -1;
          if (lim < 63) {
#pragma unroll
            for (int c = 0; c < 64; ++c) u[c] = (c > lim) ? 0xff800000u : u[c];
          }
          float m4[4] = {NEG_INF, NEG_INF, NEG_INF, NEG_INF};
#pragma unroll
          for (int c = 0; c < 64; c += 8)
#pragma unroll
            for (int q = 0; q < 4; ++q)
              m4[q] = fmax3(m4[q], __uint_as_float(u[c + 2 * q]), __uint_as_float(u[c + 2 * q + 1]));
          mh = fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3])) * sl2;  // -inf stays -inf
        }
        // ---- skip test.  BC = 128: the S tile, whose maximum is max(mA,
        // mB).  max(mA, mB) < x exactly when mA < x and mB < x, so each
        // warp votes on its own half of its rows before the exchange (the
        // running maximum m_exact is the same in the two threads of a row),
        // and the exchange's barrier makes all eight votes visible: every
        // warp reads the tile's fate without waiting for another.  BC = 64:
        // warpgroup h decides its own half, tile 2j + h, whose running
        // maximum includes half A when h = 1 (known after the exchange).
        const int di = dcount % kDR;
        const int dnum = dcount;
        ++dcount;
        const bool visited = !kHalves || 2 * j + h < it.T64;
        bool warp_pass = false;
        if constexpr (!kHalves && SKIP) {
          const bool pass = waited && (!row_valid || (m_exact != NEG_INF &&
                                                      (mh == NEG_INF || mh < m_exact - tau_log2)));
          warp_pass = __all_sync(0xffffffffu, pass) != 0;
          // every lane stores the same word (no divergent branch on the path
          // from S to P); waited is the same in every lane
          *vote_at(di, h, sw) = (dnum << 2) | (waited ? 0 : 2) | (warp_pass ? 1 : 0);
        }
        const float mo = exchange(mh);
        const float mA = h == 0 ? mh : mo;
        const float mB = h == 0 ? mo : mh;
        bool skip = false;
        if constexpr (!kHalves && SKIP) {
          // a warp with a failing row knows the tile is kept; a warp whose
          // rows all pass reads the eight votes, all in since the exchange's
          // barrier: skipped iff every warp's rows pass in both halves (a
          // warp that gave up votes keep).  Vote words [di][h][w].
          if (warp_pass) {
            int all = 1;
#pragma unroll
            for (int w = 0; w < 8; ++w) all &= vote[di * 8 + w];
            skip = (all & 1) != 0;
          }
        } else if (kHalves && SKIP) {
          const float mt = mh;
          const float mpre = h == 1 ? fmaxf(m_exact, mA) : m_exact;
          const bool pass = waited && visited &&
                            (!row_valid || (mpre != NEG_INF && (mt == NEG_INF || mt < mpre - tau_log2)));
          const bool warp_pass = __all_sync(0xffffffffu, pass) != 0;
          const bool warp_ok = waited;  // already the same in every lane (a warp vote)
          // every lane stores the same word (no divergent branch on the
          // path from S to P)
          *vote_at(di, h, sw) = (dnum << 2) | (warp_ok ? 0 : 2) | (warp_pass ? 1 : 0);
          if (warp_pass) {
            // a warp whose rows all pass learns the tile's fate from the
            // other three warps of its warpgroup (stop at the first failure)
            int verdict = 0;  // 1 keep, 2 skip, 3 gave up
            if (lane == 0) {
              const uint64_t t0 = globaltimer_ns();
              for (uint32_t n = 0; verdict == 0; ++n) {
                int n_pass = 0;
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                  const int x = *vote_at(di, h, w);
                  if ((x >> 2) == dnum) {
                    if (x & 1) ++n_pass;
                    else verdict = 1;
                  }
                }
                if (verdict == 0 && n_pass == 4) verdict = 2;
                if (verdict == 0 && (n & 15u) == 15u &&
                    (*abort_flag || globaltimer_ns() - t0 > wait_limit_ns))
                  verdict = 3;
                if (verdict == 0 && n >= 2) __nanosleep(64);
              }
            }
            verdict = __shfl_sync(0xffffffffu, verdict, 0);
            if (verdict == 3) waited = false;
            skip = verdict == 2;
          }
        }
        if (!waited) {
          // The warps run out the item (taking part in every exchange) and
          // leave together at the item-end synchronisation.
          if (!failed) give_up(abort_flag, status, 10);
          failed = true;
          continue;
        }
        if (skip_mask && row == 0 && (kHalves ? visited : h == 0))
          skip_mask[mask_base + (kHalves ? 2 * j + h : j)] = skip ? 1 : 0;
        // the exact running maximum over every visited tile (a skipped tile
        // never raises it), and the lazy reference maximum of P: both are the
        // same in the two threads of a row
        const float mtile = fmaxf(mA, mB);
        m_exact = fmaxf(m_exact, mtile);
        const float m_cand = fmaxf(m_ref, mtile);
        const bool moved = row_valid && (m_cand > m_ref + kRescale);
        float alpha = 1.f;
        if (moved) {
          alpha = ex2(m_ref - m_cand);  // 0 on the first tile (m_ref = -inf)
          m_ref = m_cand;
        }
        float rs = 0.f;
        if (!skip && visited) {
          // P = 2^(s*scale - m_ref): one packed FFMA per pair, two ex2, one
          // pack to bf16 for the P*V MMA.  The row sum adds the same
          // bf16-rounded values that the MMA multiplies, so numerator and
          // denominator see the same weights (the rounding of a dominant
          // weight cancels in O / l).
          const float neg_m = row_valid ? -m_ref : 0.f;
          const float2 nm2 = make_float2(neg_m, neg_m);
          float2 rs2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                           make_float2(0.f, 0.f)};
#pragma unroll
          for (int c0 = 0; c0 < 64; c0 += 32) {
            uint32_t pk[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const float2 x = __ffma2_rn(
                  make_float2(__uint_as_float(u[c0 + 2 * c]), __uint_as_float(u[c0 + 2 * c + 1])), sc2,
                  nm2);
              const uint32_t w = ((POLY >> c) & 1u) ? exp2_poly_bf16x2(x)
                                                          : pack_bf16x2(ex2(x.x), ex2(x.y));
              rs2[c & 3] = __fadd2_rn(rs2[c & 3], make_float2(__uint_as_float(w << 16),
                                                              __uint_as_float(w & 0xffff0000u)));
              pk[c] = w;
            }
            tmem_st16(tS(sb) + h * 64 + lane_off + c0 / 2, pk);
          }
          const float2 rsa = __fadd2_rn(__fadd2_rn(rs2[0], rs2[1]), __fadd2_rn(rs2[2], rs2[3]));
          rs = rsa.x + rsa.y;
        }
        l_h = l_h * alpha + rs;
        // O rescale: this warpgroup's 64 columns of O, once P*V of S tile
        // j - 1 has finished (commit #(base + pro + j - 1))
        if (j > 0 && __any_sync(0xffffffffu, moved)) {
          if (!__all_sync(0xffffffffu, wait_cm(base + pro + j - 1))) {
            give_up(abort_flag, status, 12);
            failed = true;  // acted on at the item end
          } else {
            tc_fence_after();
            const float a = moved ? alpha : 1.f;
#pragma unroll
            for (int c0 = 0; c0 < 64; c0 += 32) {
              uint32_t r[32];
              tmem_ld32(tO + lane_off + h * 64 + c0, r);
              tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < 32; ++c) r[c] = __float_as_uint(__uint_as_float(r[c]) * a);
              tmem_st32(tO + lane_off + h * 64 + c0, r);
            }
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(b_p_full(sb));
        // the previous item's O store has had a tile's time to read its Q slot
        if (j == 0 && row == 0) release_pending();
      }
      // ---- epilogue: tiles not visited are marked 2; O / l -> bf16 -> TMA store
      if (skip_mask && h == 0)
        for (int t = (kHalves ? it.T64 : it.T) + row; t < n_dec; t += kRows) skip_mask[mask_base + t] = 2;
      // P*V of the last tile finished: commit #(base + pro + T - 1).  Give-ups
      // of any warp during the item are combined over all eight softmax
      // warps, which then go on, or leave, together.
      bool done = !failed && __all_sync(0xffffffffu, wait_cm(base + pro + it.T - 1));
      base += pro + it.T;
      volatile int* lv = leave + (leaves & 1) * 8;
      ++leaves;
      if (lane == 0) lv[warp - 4] = done ? 0 : 1;
      const float l_o = exchange(l_h);  // the barrier also publishes the leave flags
#pragma unroll
      for (int w = 0; w < 8; ++w)
        if (lv[w]) done = false;
      if (!done) {
        if (!failed) give_up(abort_flag, status, 11);
        ok = false;
        break;
      }
      tc_fence_after();
      const float l = h == 0 ? l_h + l_o : l_o + l_h;  // the same sum in both threads
      const float inv_l = row_valid ? 1.f / l : 0.f;
      // Stage this warpgroup's 64 columns of O (bf16, TMA layout: one
      // 64-column panel, 128-byte swizzle) in panel h of the item's Q slot,
      // which no MMA reads any more (its last S MMA completed before the last
      // P*V); then one thread stores the panel.  Rows past N are clipped.
      const uint32_t stage = sQ + qs * kTile + h * kPanel;
#pragma unroll
      for (int c0 = 0; c0 < 64; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(tO + lane_off + h * 64 + c0, r);
        tmem_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int c = 0; c < 16; ++c)
          w[c] = pack_bf16x2(__uint_as_float(r[2 * c]) * inv_l, __uint_as_float(r[2 * c + 1]) * inv_l);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int lc = c0 / 8 + q;  // 16-byte chunk of the panel row
          const uint32_t a = stage + row * 128 + (((lc & 7) ^ (row & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(w[4 * q]),
                       "r"(w[4 * q + 1]), "r"(w[4 * q + 2]), "r"(w[4 * q + 3])
                       : "memory");
        }
      }
      fence_proxy_async_smem();  // the generic-proxy writes, before the async-proxy store
      named_bar(2 + h, 128);
      if (row == 0) {
        release_pending();  // at most one store in flight per warpgroup
        tma_store_3d(&tmO, stage, h * 64, it.rb * kRows, it.bh);
        bulk_commit_group();
        pend_slot = qs;
      }
      // O may be overwritten by the next item's first P*V only after both
      // warpgroups signal that item's first P: ordering comes from p_full
      tc_fence_before();
    }
    // no store may still be reading shared memory, or writing O, at exit
    if (row == 0) {
      release_pending();
      bulk_wait_all();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// --------------------------------------------------------------------- host
namespace {

template <int BC, bool CAUSAL, uint32_t POLY, bool SKIP>
int split_launch_t(const PrefillLaunch& a) {
  auto kern = prefill_split_kernel<BC, CAUSAL, POLY, SKIP>;
  static uint64_t ready = 0;  // one bit per device: attributes set and checked
  static int sm_count[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return ATTN_ERR_CUDA;
  if (!(ready >> dev & 1)) {
    // The register split (setmaxnreg) assumes exactly kRegs registers per
    // thread at launch; anything else could leave setmaxnreg.inc waiting.
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return ATTN_ERR_CUDA;
    if (fa.numRegs != kRegs) return ATTN_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) !=
        cudaSuccess)
      return ATTN_ERR_CUDA;
    if (cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return ATTN_ERR_CUDA;
    ready |= uint64_t(1) << dev;
  }
  CUtensorMap mq, mk, mv, mo;
  if (!tma_map_bhnd(&mq, a.Q, a.B * a.Hq, a.N, kD, kRows) ||
      !tma_map_bhnd(&mk, a.K, a.B * a.Hkv, a.N, kD, kST) ||
      !tma_map_bhnd(&mv, a.V, a.B * a.Hkv, a.N, kD, BC) ||
      !tma_map_bhnd(&mo, a.O, a.B * a.Hq, a.N, kD, kRows))
    return ATTN_ERR_CUDA;
  const long long n_items = static_cast<long long>(a.B) * a.Hq * ((a.N + kRows - 1) / kRows);
  const int grid = static_cast<int>(n_items < sm_count[dev] ? n_items : sm_count[dev]);
  kern<<<grid, kThreads, kSmemBytes, a.stream>>>(mq, mk, mv, mo, a.skip_mask, a.status, a.B, a.Hq,
                                                 a.Hkv, a.N, a.scale_log2, a.tau_log2, a.wait_limit_ns);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <int BC, bool CAUSAL, uint32_t POLY>
int split_launch(const PrefillLaunch& a) {
  return a.tau_is_inf ? split_launch_t<BC, CAUSAL, POLY, false>(a) : split_launch_t<BC, CAUSAL, POLY, true>(a);
}

}  // namespace

int launch_prefill_split(const PrefillLaunch& a) {
  if (a.Br != 128 || a.d != 128 || a.cu_seqlens || a.q_scales) return ATTN_ERR_INVALID_ARG;
  if (a.poly_pairs != 0) {  // polynomial exp2 on 4 or 8 of every 16 pairs; Bc = 128
    if (a.Bc != 128) return ATTN_ERR_INVALID_ARG;
    if (a.poly_pairs == 4)
      return a.causal ? split_launch<128, true, 0x1111u>(a) : split_launch<128, false, 0x1111u>(a);
    if (a.poly_pairs == 8)
      return a.causal ? split_launch<128, true, 0x5555u>(a) : split_launch<128, false, 0x5555u>(a);
    return ATTN_ERR_INVALID_ARG;
  }
  if (a.Bc == 64) return a.causal ? split_launch<64, true, 0>(a) : split_launch<64, false, 0>(a);
  if (a.Bc == 128) return a.causal ? split_launch<128, true, 0>(a) : split_launch<128, false, 0>(a);
  return ATTN_ERR_INVALID_ARG;
}

}  // namespace bss
