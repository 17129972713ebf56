// Skip Softmax prefill for sm_100a, two row blocks per CTA ("ping-pong"),
// persistent over work items.  Used for Br = 128.
//
// Method: "Accelerating Long-Context Inference with Skip Softmax in NVIDIA
// TensorRT-LLM" (Key Points; Detailed Analysis): key tiles in ascending
// order; tile j of a row block is skipped -- no exponentials, no P*V MMA --
// iff every row of that row block has tile max < running max - tau.  The V
// tile is loaded iff at least one of the CTA's two row blocks keeps it.
//
// Layout of one CTA (384 threads, one per SM, persistent):
//   warpgroup 0: warp 0 TMA Q (both tiles) + K ring; warp 1 TMEM allocator
//                and an MMA-issuing thread; warp 2 TMA V ring (gated by the
//                skip decisions); warp 3 the second MMA-issuing thread
//                (tau = inf with two S buffers per row block: one issuer per
//                row block), else idle.
//   warpgroup 1: softmax of row block 0 (thread r owns row r).
//   warpgroup 2: softmax of row block 1.
// TMEM (512 columns): O0 | O1 | S/P buffers (two per row block when Bc = 64,
// one when Bc = 128), P_t (bf16) written over S_t.
// MMA issue order per key tile j and row block t:  PV_t_j, S_t_{j+SB}, commit
// so the exponentials of one row block overlap the other block's MMAs.  The
// tcgen05 issue queue holds only a few MMAs, so an issuing thread stalls at
// the pipe's pace; with a single issuer, each of its waits (for one row
// block's P, or for K or V) lets the pipe run dry, which is why each row
// block gets its own issuer where the loads allow it.
//
// Completion signalling.  Each issuer makes exactly one commit per row block
// and step (plus the first SB S tiles of a work item and one Q-slot release
// per item), into a ring of mbarriers per row block indexed by a running
// commit count.  Every completion that a role needs is one of those commits:
//   S_t of key tile i ready         commit #(base_t + i)
//   P*V_t of key tile j finished    commit #(base_t + min(SB, T_t) + j)
// (a commit covers every earlier MMA of the thread that issues it, and one
// thread issues all of a row block's MMAs).  K and V ring slots wait for the
// commits of every row block that reads them; the O rescale and the epilogue
// wait on their own row block's.  Every wait is bounded; a wait that gives
// up records a status code and the CTA unwinds (leaving no copy or MMA in
// flight and freeing TMEM).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "exp2_poly.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace bss {

namespace {

constexpr int kPPThreads = 384;
constexpr int kPPRegs = 168;  // registers per thread at launch (checked on the host)
constexpr int kRows = 128;    // rows per tile (row block)
constexpr int kDR = 4;        // decision ring
constexpr float kI2FOffset = 12582912.f;  // 1.5 * 2^23: int32 scores as fp32 by one integer add
constexpr int kCR = 16;       // commit ring per row block (waiters lag by at most ~6)
constexpr float kRescale = 8.0f;  // lazy rescale threshold (log2 units)
// Which of the 16 column pairs of each 32-column chunk take the polynomial
// exp2 instead of MUFU (bit c = pair c).  Measured on B200 the softmax here is
// not bound by MUFU throughput, and every fraction tried (1/4 to 3/4) made
// this kernel slower, so it takes none; the column-split kernel offers the
// polynomial through attn_prefill_poly.
constexpr uint32_t kPolyPairs = 0x0000u;



// QK8: Q and K arrive as e4m3 (one byte per element, 128-byte rows hold 128
// columns) and S = Q K^T runs as kind::f8f6f4 MMAs; V and P stay bf16.
template <int D, int BC, bool QK8 = false>
struct PPCfg {
  static constexpr int kEB = QK8 ? 1 : 2;                 // bytes per Q/K element
  static constexpr int kQKPanels = D * kEB / 128;        // 128-byte column panels of Q and K
  static constexpr int kVPanels = D / 64;                // of V (bf16)
  static constexpr int kQKCols = 128 / kEB;              // Q/K columns per panel
  static constexpr int kSSteps = D * kEB / 32;           // S MMAs per tile (32 bytes of K each)
  static constexpr int kQTile = kRows * D * kEB;
  static constexpr int kQPanel = kRows * 128;
  static constexpr int kKBytes = BC * D * kEB;
  static constexpr int kVBytes = BC * D * 2;
  static constexpr int kKVPanel = BC * 128;
  static constexpr int kKS = (BC == 128 && D == 128 && !QK8) ? 2 : 3;
  static constexpr int kVS = (BC == 128 && D == 128 && !QK8) ? 2 : 3;
  // S/P buffers per row block: two when TMEM has room (Bc = 64), so the MMA
  // for key tile j+1 runs while the softmax works on tile j
  static constexpr int kSB = (2 * D + 4 * BC <= 512) ? 2 : 1;
  // Q slots: with two, the next work item's Q loads while this one runs
  static constexpr int kQS = (BC == 128 && D == 128 && !QK8) ? 1 : 2;
  static constexpr int kQSlot = 2 * kQTile;  // two row blocks
  // With two Q slots, a row block's O is staged in its own (finished) Q tile
  // and written by a TMA store; the slot is released once the store has read
  // it.  An e4m3 Q tile is too small to hold the bf16 O tile: there, where
  // shared memory has room (the e4m3 Q slots take half the bytes), each row
  // block stages O in a tile of its own (kOSep) and the Q slot is released by
  // the MMAs as without the TMA store.
  static constexpr int kOTile = kRows * D * 2;
  static constexpr bool kOSep =
      QK8 && kQS == 2 &&
      kQS * kQSlot + kKS * kKBytes + kVS * kVBytes + 2 * kOTile + 4096 <= 227 * 1024;
  static constexpr bool kTmaEpi = kQS == 2 && (!QK8 || kOSep);
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQS * kQSlot;
  static constexpr int kOffV = kOffK + kKS * kKBytes;
  static constexpr int kOffO = kOffV + kVS * kVBytes;
  static constexpr int kOffBar = kOffO + (kOSep ? 2 * kOTile : 0);
  // k_full[KS], v_full[VS], commit ring[2][CR], p_full[2][SB],
  // q_full[QS], q_empty[QS], mma_done[2]
  static constexpr int kNumBars = kKS + kVS + 2 * kCR + 2 * kSB + 2 * kQS + 2;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 256 + 1024;
  static constexpr int kTmemCols = 512;
  // setmaxnreg split of the 384 x 168 launch registers: 128 producer threads
  // (TMA, MMA issue) and 256 softmax threads; at 72 the MMA issuer does not spill
  static constexpr int kProducerRegs = 72;
  static constexpr int kSoftmaxRegs = (kPPThreads * kPPRegs - 128 * kProducerRegs) / 256 / 8 * 8;
  static_assert(128 * kProducerRegs + 256 * kSoftmaxRegs <= kPPThreads * kPPRegs, "register split");
  static_assert(2 * D + 2 * kSB * BC <= 512, "TMEM budget");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static_assert(kKS + kSB + 1 < kCR && kVS + kSB + 1 < kCR, "commit ring too small");
};

struct PPMisc {
  uint32_t tmem_base;
  int abort;
  // vote[t][i][w]: (decision number << 2) | 2 if warp w of row block t gave
  // up | 1 if every row of that warp passes the skip test, for the decision
  // in ring slot i (the decision number runs over all key tiles a row block
  // visits).  The tile is skipped iff all four warps pass.
  int vote[2][kDR][4];
  int leave[2][2][4];
};


__device__ __forceinline__ void pp_give_up(PPMisc* m, int* status, int where) {
  reinterpret_cast<volatile int*>(&m->abort)[0] = 1;
  atomicCAS(status, 0, ATTN_DEVICE_TIMEOUT_BASE + 32 + where);
}

// Work item -> (bh, pair).  Causal: longest pairs first, heads fastest.
// Non-causal: pairs fastest, so CTAs reading one head's K/V run together.
// Variable-length batches (VARLEN): N is the longest sequence; items run
// over (pair, sequence, head), longest pairs first, and a pair past the end
// of its sequence is an empty item (T0 = 0) that every role skips.
struct Item {
  int bh, rb0, T0, T1, Tmax;  // T1 = 0 when the second row block does not exist
  int len, tok0;              // keys of this sequence, and its first token (VARLEN)
};

template <int BC, bool CAUSAL, bool VARLEN>
__device__ __forceinline__ Item make_item(long long idx, int BH, int n_pairs, int n_rb, int N,
                                          int Hq, int Hkv, bool group_major, const int* cu_seqlens,
                                          int total) {
  Item it;
  int pair;
  if (VARLEN) {
    pair = n_pairs - 1 - static_cast<int>(idx / BH);
    it.bh = static_cast<int>(idx % BH);
    const int b = it.bh / Hq;
    // clamped, so that a malformed cu_seqlens cannot move a row past the tensors
    it.tok0 = min(max(cu_seqlens[b], 0), total);
    it.len = max(0, min(min(N, cu_seqlens[b + 1] - it.tok0), total - it.tok0));
  } else if (CAUSAL && group_major) {
    // KV-head groups one after another (longest pairs first inside a group,
    // heads fastest): the CTAs in flight share one group's K/V, which then
    // stays in L2 however long the sequence
    const int g = Hq / Hkv;
    const long long per_group = static_cast<long long>(g) * n_pairs;
    const int grp = static_cast<int>(idx / per_group);
    const int r = static_cast<int>(idx % per_group);
    pair = n_pairs - 1 - r / g;
    it.bh = grp * g + r % g;
    it.len = N;
    it.tok0 = 0;
  } else if (CAUSAL) {
    pair = n_pairs - 1 - static_cast<int>(idx / BH);
    it.bh = static_cast<int>(idx % BH);
    it.len = N;
    it.tok0 = 0;
  } else {
    pair = static_cast<int>(idx % n_pairs);
    it.bh = static_cast<int>(idx / n_pairs);
    it.len = N;
    it.tok0 = 0;
  }
  it.rb0 = 2 * pair;
  if constexpr (VARLEN) {
    const int n_tiles = (it.len + BC - 1) / BC;
    const int n_rb_s = (it.len + kRows - 1) / kRows;
    auto visited = [&](int rb) {
      if (rb >= n_rb_s) return 0;
      const int last = min(it.len, (rb + 1) * kRows) - 1;
      return CAUSAL ? (last / BC + 1) : n_tiles;
    };
    it.T0 = visited(it.rb0);
    it.T1 = visited(it.rb0 + 1);
  } else {
    const int n_tiles = (N + BC - 1) / BC;
    auto visited = [&](int rb) {
      const int last = min(N, (rb + 1) * kRows) - 1;
      return CAUSAL ? (last / BC + 1) : n_tiles;
    };
    it.T0 = visited(it.rb0);
    it.T1 = (it.rb0 + 1 < n_rb) ? visited(it.rb0 + 1) : 0;
  }
  it.Tmax = max(it.T0, it.T1);
  return it;
}

// Commits a row block makes in one work item: its first SB S tiles, then one
// per key tile it visits.
template <int SB>
__device__ __forceinline__ int commits_of(int T) { return T > 0 ? min(SB, T) + T : 0; }

// A short FIFO of ring-slot releases: (row block, commit index) that must
// complete before the slot's next copy.  Fixed positions keep it in registers.
// The tile number g (running over work items) says when a wait is not needed.
// A ring slot's last tile: the commit numbers of row blocks 0 and 1 that
// cover its reads (-1: that row block does not read it), and its running
// tile number g.
struct Pending3 {
  int c0[3], c1[3], g[3], n;
  __device__ __forceinline__ void init() { n = 0; }
  // constant indices keep the entries in registers
  __device__ __forceinline__ void push(int cc0, int cc1, int gg) {
    if (n == 0) { c0[0] = cc0; c1[0] = cc1; g[0] = gg; }
    else if (n == 1) { c0[1] = cc0; c1[1] = cc1; g[1] = gg; }
    else { c0[2] = cc0; c1[2] = cc1; g[2] = gg; }
    ++n;
  }
  __device__ __forceinline__ void pop() {
    c0[0] = c0[1]; c1[0] = c1[1]; g[0] = g[1];
    c0[1] = c0[2]; c1[1] = c1[2]; g[1] = g[2];
    --n;
  }
};

}  // namespace

// QKT: Q K^T operand format, 0 bf16, 1 e4m3 (f32 scores), 2 signed int8
// (int32 scores).  SKIP: tau is finite, so the kernel takes the skip test;
// with tau = inf it holds no trace of it (the test's branches alone cost the
// softmax loop several per cent in scheduling).
template <int D, int BC, bool CAUSAL, bool VARLEN, int QKT, bool SKIP>
__global__ void __launch_bounds__(kPPThreads, 1)
    prefill_pp_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                      __nv_bfloat16* __restrict__ O,
                      uint8_t* __restrict__ skip_mask, int* __restrict__ status, int B, int Hq,
                      int Hkv, int N, float scale_log2, float tau_log2,
                      unsigned long long wait_limit_ns, const int* __restrict__ cu_seqlens,
                      int total, const float* __restrict__ q_scales,
                      const float* __restrict__ k_scales) {
  constexpr bool QK8 = QKT != 0;
  using C = PPCfg<D, BC, QK8>;
  // variable-length batches store O row by row: a TMA store of the last row
  // block would write into the next sequence's rows
  // O by TMA store (variable-length batches: row blocks that end inside
  // their sequence; the last, partial one of a sequence stores row by row)
  constexpr bool kTmaEpi = C::kTmaEpi;
  constexpr bool kOSep = C::kOSep && !VARLEN;  // O staged apart from the Q slot
  constexpr int SB = C::kSB;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + C::kOffQ;
  const uint32_t sK = sbase + C::kOffK;
  const uint32_t sV = sbase + C::kOffV;
  const uint32_t bar0 = sbase + C::kOffBar;
  auto b_k_full = [&](int s) { return bar0 + 8u * s; };
  auto b_v_full = [&](int s) { return bar0 + 8u * (C::kKS + s); };
  constexpr int kBC = C::kKS + C::kVS;
  auto b_cm = [&](int t, int i) { return bar0 + 8u * (kBC + t * kCR + (i % kCR)); };
  constexpr int kBP = kBC + 2 * kCR;
  auto b_p_full = [&](int t, int b) { return bar0 + 8u * (kBP + t * SB + b); };
  constexpr int kBQ = kBP + 2 * SB;
  auto b_q_full = [&](int s) { return bar0 + 8u * (kBQ + s); };
  auto b_q_empty = [&](int s) { return bar0 + 8u * (kBQ + C::kQS + s); };
  // mma_done of MMA issuer 0 and 1 (two issuers at tau = inf)
  auto b_mma_done = [&](int i) { return bar0 + 8u * (kBQ + 2 * C::kQS + i); };
  // With tau = inf every V tile is loaded, so tile j of an item is V load
  // number (tiles of earlier items) + j for both row blocks: each row block
  // then gets an MMA issuer of its own (warps 1 and 3).  The tcgen05 issue
  // queue is a few MMAs deep, so a single issuer's waits for one row block
  // let the pipe run dry while the other row block's work is ready.  With a
  // finite tau the V loads depend on both row blocks' decisions and warp 1
  // issues for both.  With one S buffer per row block (Bc = 128 at d = 128)
  // the single issuer's fixed alternation measured faster, so it stays.
  constexpr bool dual = !SKIP && SB == 2;
  PPMisc* misc = reinterpret_cast<PPMisc*>(smem + C::kOffMisc);
  volatile int* abort_flag = &misc->abort;
  // keep (1) or skip (0) from the four vote words of one decision
  auto decided_keep = [&](int t, int i) -> int {
    const volatile int* v = misc->vote[t][i];
    return ((v[0] & v[1] & v[2] & v[3]) & 1) ? 0 : 1;
  };
  // all four votes of row block t for decision number dnum (ring slot i)
  // are in; false if the wait gave up (the abort flag, or the time limit)
  auto votes_in = [&](int t, int i, int dnum) -> bool {
    const volatile int* v = misc->vote[t][i];
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t n = 0;; ++n) {
      if ((v[0] >> 2) == dnum && (v[1] >> 2) == dnum && (v[2] >> 2) == dnum && (v[3] >> 2) == dnum)
        return true;
      if ((n & 15u) == 15u && (*abort_flag || globaltimer_ns() - t0 > wait_limit_ns)) return false;
      __nanosleep(96);
    }
  };
  // wait for commit number i of row block t (bounded)
  auto wait_cm = [&](int t, int i) {
    return mbar_wait(b_cm(t, i), (i / kCR) & 1, abort_flag, wait_limit_ns);
  };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_rb = (N + kRows - 1) / kRows;
  const int n_pairs = (n_rb + 1) / 2;
  const int BH = B * Hq;
  const int g = Hq / Hkv;
  const int n_tiles = (N + BC - 1) / BC;
  const long long n_items = static_cast<long long>(BH) * n_pairs;
  // The k-th work item of this CTA: items go out in rounds of gridDim.x.
  // Causal items are numbered longest first and go out in a "snake": CTAs in
  // ascending order in even rounds and descending in odd ones, which evens
  // out the work per CTA (for the causal 8B layer the busiest CTA had 14 %
  // more than the mean with plain round robin, 1.6 % with the snake).
  // Non-causal items are all equal and keep plain round robin.  Once an index
  // passes n_items every later one does too.
  // Causal layers whose KV-head groups hold many items per CTA (long
  // sequences) go group by group, so the K/V read by the CTAs in flight fits
  // in L2 (the 128K-token 70B layer: 537 MB of K/V in all, 67 MB per group);
  // with few items per group, rounds of one group would mix long and short
  // items and unbalance the CTAs, so heads stay fastest there.
  const bool group_major =
      CAUSAL && !VARLEN && static_cast<long long>(g) * n_pairs >= 8LL * gridDim.x;
  auto item_idx = [&](long long k) -> long long {
    const long long G = gridDim.x;
    return k * G + ((CAUSAL && (k & 1)) ? G - 1 - blockIdx.x : blockIdx.x);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kKS; ++s) mbar_init(b_k_full(s), 1);
    for (int s = 0; s < C::kVS; ++s) mbar_init(b_v_full(s), 1);
    for (int t = 0; t < 2; ++t) {
      for (int i = 0; i < kCR; ++i) mbar_init(b_cm(t, i), 1);
      for (int b = 0; b < SB; ++b) mbar_init(b_p_full(t, b), 4);
    }
    for (int s = 0; s < C::kQS; ++s) {
      mbar_init(b_q_full(s), 1);
      // one arrival per row block's O store, or per MMA issuer
      mbar_init(b_q_empty(s), (kTmaEpi && !kOSep) || dual ? 2 : 1);
    }
    mbar_init(b_mma_done(0), 1);
    mbar_init(b_mma_done(1), 1);
    for (int t = 0; t < 2; ++t)
      for (int i = 0; i < kDR; ++i)
        for (int w = 0; w < 4; ++w) misc->vote[t][i][w] = -1;  // no decision number matches
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
  auto tO = [&](int t) { return tmem + t * D; };
  auto tS = [&](int t, int b) { return tmem + 2 * D + (t * SB + b) * BC; };

  if (warp < 4) {
    reg_dec<C::kProducerRegs>();
    if (warp == 0 && lane == 0) {
      // ---------------------------------------------------- Q and K producer
      int kload = 0, items = 0, kdone = 0;
      int base0 = 0, base1 = 0;  // commit counts of earlier items, per row block
      Pending3 pend;
      pend.init();
      bool alive = true;
      // items counts the non-empty work items (their Q slots); k every index
      for (long long k = 0, idx = item_idx(0); alive && idx < n_items; idx = item_idx(++k)) {
        const Item it = make_item<BC, CAUSAL, VARLEN>(idx, BH, n_pairs, n_rb, N, Hq, Hkv, group_major, cu_seqlens, total);
        if (VARLEN && it.T0 == 0) continue;  // a pair past the end of its sequence
        const int bkv = (it.bh / Hq) * Hkv + (it.bh % Hq) / g;
        const int qs = items % C::kQS;
        if (items >= C::kQS && !mbar_wait(b_q_empty(qs), ((items / C::kQS) - 1) & 1, abort_flag,
                                          wait_limit_ns)) {
          pp_give_up(misc, status, 1);
          break;
        }
        const int nq = it.T1 > 0 ? 2 : 1;
        mbar_arrive_expect_tx(b_q_full(qs), nq * C::kQTile);
        for (int t = 0; t < nq; ++t)
          for (int p = 0; p < C::kQKPanels; ++p)
            if constexpr (VARLEN)  // Q as [tokens, Hq, d]
              tma_load_3d(sQ + qs * C::kQSlot + t * C::kQTile + p * C::kQPanel, &tmQ, b_q_full(qs),
                          p * C::kQKCols, it.bh % Hq, it.tok0 + (it.rb0 + t) * kRows);
            else
              tma_load_3d(sQ + qs * C::kQSlot + t * C::kQTile + p * C::kQPanel, &tmQ, b_q_full(qs),
                          p * C::kQKCols, (it.rb0 + t) * kRows, it.bh);
        for (int j = 0; j < it.Tmax; ++j) {
          const int s = kload % C::kKS;
          if (pend.n == C::kKS) {  // the slot's previous tile: its S MMAs must have run
            if ((pend.c0[0] >= 0 && !wait_cm(0, pend.c0[0])) ||
                (pend.c1[0] >= 0 && !wait_cm(1, pend.c1[0]))) {
              pp_give_up(misc, status, 2);
              alive = false;
              break;
            }
            pend.pop();
          }
          mbar_arrive_expect_tx(b_k_full(s), C::kKBytes);
          for (int p = 0; p < C::kQKPanels; ++p) {
            if constexpr (VARLEN)  // K as [tokens, Hkv, d]
              tma_load_3d(sK + s * C::kKBytes + p * C::kKVPanel, &tmK, b_k_full(s), p * C::kQKCols,
                          (it.bh % Hq) / g, it.tok0 + j * BC);
            else
              tma_load_3d(sK + s * C::kKBytes + p * C::kKVPanel, &tmK, b_k_full(s), p * C::kQKCols,
                          j * BC, bkv);
          }
          // K tile j is read by S_j of each row block that visits it; with
          // one MMA issuer, row block 1's (if it visits j: T1 >= T0) is last
          if (dual)
            pend.push(j < it.T0 ? base0 + j : -1, j < it.T1 ? base1 + j : -1, 0);
          else if (j < it.T1)
            pend.push(-1, base1 + j, 0);
          else
            pend.push(base0 + j, -1, 0);
          ++kload;
        }
        base0 += commits_of<SB>(it.T0);
        base1 += commits_of<SB>(it.T1);
        kdone = items + 1;
        ++items;
      }
      // never leave with a copy in flight
      for (int i = max(0, kdone - C::kQS); i < kdone; ++i)
        mbar_drain(b_q_full(i % C::kQS), (i / C::kQS) & 1, wait_limit_ns);
      for (int t = max(0, kload - C::kKS); t < kload; ++t)
        mbar_drain(b_k_full(t % C::kKS), (t / C::kKS) & 1, wait_limit_ns);
    } else if (warp == 2 && lane == 0) {
      // ---------------------------------------------------- V producer
      int vload = 0;
      int dl[2] = {0, 0};
      int base0 = 0, base1 = 0;
      int gbase = 0;  // running tile number of this item's key tile 0
      Pending3 pend;
      pend.init();
      bool alive = true;
      for (long long k = 0, idx = item_idx(0); alive && idx < n_items; idx = item_idx(++k)) {
        const Item it = make_item<BC, CAUSAL, VARLEN>(idx, BH, n_pairs, n_rb, N, Hq, Hkv, group_major, cu_seqlens, total);
        if (VARLEN && it.T0 == 0) continue;  // a pair past the end of its sequence
        const int bkv = (it.bh / Hq) * Hkv + (it.bh % Hq) / g;
        const int T[2] = {it.T0, it.T1};
        auto issue_v = [&](int j) -> bool {
          if (pend.n == C::kVS) {
            // The slot's previous tile: its P*V MMAs must have run.  Once a
            // decision on tile j has been read, S_j has completed, and with
            // it every MMA issued before it: all P*V of tiles j - SB - 1 and
            // earlier (items are SB apart in g).  Those commits are not
            // waited for, since their ring slot may have been reused after a
            // run of skipped tiles.
            const bool known_done = SKIP && pend.g[0] + SB < gbase + j;
            if (!known_done && ((pend.c0[0] >= 0 && !wait_cm(0, pend.c0[0])) ||
                                (pend.c1[0] >= 0 && !wait_cm(1, pend.c1[0]))))
              return false;
            pend.pop();
          }
          const int s = vload % C::kVS;
          mbar_arrive_expect_tx(b_v_full(s), C::kVBytes);
          for (int p = 0; p < C::kVPanels; ++p) {
            if constexpr (VARLEN)  // V as [tokens, Hkv, d]
              tma_load_3d(sV + s * C::kVBytes + p * C::kKVPanel, &tmV, b_v_full(s), p * 64,
                          (it.bh % Hq) / g, it.tok0 + j * BC);
            else
              tma_load_3d(sV + s * C::kVBytes + p * C::kKVPanel, &tmV, b_v_full(s), p * 64, j * BC,
                          bkv);
          }
          // P*V of tile j by each row block that visits it; with one MMA
          // issuer, row block 1's (if it visits j) is issued after row block 0's
          if (dual)
            pend.push(j < it.T0 ? base0 + min(SB, it.T0) + j : -1,
                      j < it.T1 ? base1 + min(SB, it.T1) + j : -1, gbase + j);
          else if (j < it.T1)
            pend.push(-1, base1 + min(SB, it.T1) + j, gbase + j);
          else
            pend.push(base0 + min(SB, it.T0) + j, -1, gbase + j);
          ++vload;
          return true;
        };
        for (int j = 0; alive && j < it.Tmax; ++j) {
          if (!SKIP) {
            if (!issue_v(j)) {
              pp_give_up(misc, status, 4);
              alive = false;
            }
            continue;
          }
          // V_j is loaded as soon as either row block keeps tile j; every
          // decision is still consumed, in order
          bool issued = false;
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            if (!alive || j >= T[t]) continue;
            // the softmax warps publish their votes without a barrier
            // arrival (an arrival is a long-latency step on their path from
            // S to P); this thread polls the four vote words of decision
            // dl[t] of row block t, with a bounded wait
            const int di = dl[t] % kDR;
            if (!votes_in(t, di, dl[t])) {
              pp_give_up(misc, status, 3);
              alive = false;
              continue;
            }
            ++dl[t];
            if (decided_keep(t, di) && !issued) {
              if (!issue_v(j)) {
                pp_give_up(misc, status, 4);
                alive = false;
                continue;
              }
              issued = true;
            }
          }
        }
        base0 += commits_of<SB>(it.T0);
        base1 += commits_of<SB>(it.T1);
        gbase += it.Tmax + SB;
      }
      for (int t = max(0, vload - C::kVS); t < vload; ++t)
        mbar_drain(b_v_full(t % C::kVS), (t / C::kVS) & 1, wait_limit_ns);
    } else if ((warp == 1 || (warp == 3 && dual)) && lane == 0) {
      // ---------------------------------------------------- MMA issuer(s)
      constexpr uint32_t idS = QKT == 2   ? idesc_s8_s32(kRows, BC)
                               : QKT == 1 ? idesc_e4m3_f32(kRows, BC)
                                          : idesc_bf16_f32(kRows, BC, false, false);
      constexpr uint32_t idPV = idesc_bf16_f32(kRows, D, false, true);
      int kuse = 0, vuse = 0, items = 0;
      int pc[2] = {0, 0}, dc[2] = {0, 0}, sq[2] = {0, 0}, cmc[2] = {0, 0};
      bool alive = true;
      // Descriptors differ only in their start-address field (bits 0-13, in
      // 16-byte units): each MMA adds a compile-time offset to a 32-bit base.
      constexpr uint32_t kHi = sw128_desc_hi(1024);
      const uint32_t dK0 = sw128_desc_lo(sK, 16);
      const uint32_t dV0 = sw128_desc_lo(sV, C::kKVPanel);
      uint32_t dQ = sw128_desc_lo(sQ, 16);  // this item's Q slot
      auto issue_S = [&](int t, int kslot, int buf) {
        const uint32_t a0 = dQ + t * (C::kQTile >> 4);
        const uint32_t b0 = dK0 + kslot * (C::kKBytes >> 4);
#pragma unroll
        for (int kk = 0; kk < C::kSSteps; ++kk) {  // 32 bytes of the reduction each
          const uint32_t oq = ((kk >> 2) * C::kQPanel + (kk & 3) * 32) >> 4;
          const uint32_t ok_ = ((kk >> 2) * C::kKVPanel + (kk & 3) * 32) >> 4;
          if constexpr (QKT == 2)
            mma_ss_i8(tS(t, buf), desc_join(a0 + oq, kHi), desc_join(b0 + ok_, kHi), idS,
                      kk > 0 ? 1u : 0u);
          else if constexpr (QKT == 1)
            mma_ss_f8(tS(t, buf), desc_join(a0 + oq, kHi), desc_join(b0 + ok_, kHi), idS,
                      kk > 0 ? 1u : 0u);
          else
            mma_ss(tS(t, buf), desc_join(a0 + oq, kHi), desc_join(b0 + ok_, kHi), idS,
                   kk > 0 ? 1u : 0u);
        }
      };
      auto commit = [&](int t) {
        mma_commit(b_cm(t, cmc[t]));
        ++cmc[t];
      };
      const int me = warp == 1 ? 0 : 1;  // the issuer's done barrier (and row block, when dual)
      if (dual) {
        // One row block per issuer.  K tile j of an item is K load number
        // kbase + j (every tile of every item is loaded), and at tau = inf
        // V tile j is V load number kbase + j as well.  Each row block's
        // commits keep the single-issuer numbering: min(SB, T) for the
        // first S tiles, then one per key tile (P*V_j and S_{j+SB}).
        const int t = me;
        long long kbase = 0;
        // scalars: a runtime index into the per-row-block arrays would put
        // them in local memory
        int pcm = 0, sqm = 0, cmm = 0;
        auto commit_me = [&]() {
          mma_commit(b_cm(t, cmm));
          ++cmm;
        };
        for (long long k = 0, idx = item_idx(0); alive && idx < n_items; idx = item_idx(++k)) {
          const Item it = make_item<BC, CAUSAL, VARLEN>(idx, BH, n_pairs, n_rb, N, Hq, Hkv, group_major, cu_seqlens, total);
          if (VARLEN && it.T0 == 0) continue;  // a pair past the end of its sequence
          const int T = t == 0 ? it.T0 : it.T1;
          const int qs = items % C::kQS;
          ++items;
          if (T == 0) {  // this row block does not exist: its share of the Q slot release
            if (!kTmaEpi || kOSep) mbar_arrive(b_q_empty(qs));
            kbase += it.Tmax;
            continue;
          }
          dQ = sw128_desc_lo(sQ + qs * C::kQSlot, 16);
          if (!mbar_wait(b_q_full(qs), ((items - 1) / C::kQS) & 1, abort_flag, wait_limit_ns)) {
            pp_give_up(misc, status, 5);
            break;
          }
          auto wait_k = [&](long long g) -> bool {
            if (!mbar_wait(b_k_full(static_cast<int>(g % C::kKS)), static_cast<int>(g / C::kKS) & 1,
                           abort_flag, wait_limit_ns)) {
              pp_give_up(misc, status, 6);
              return false;
            }
            tc_fence_after();
            return true;
          };
          for (int jj = 0; jj < SB && jj < T; ++jj) {  // S of the first SB key tiles
            if (!wait_k(kbase + jj)) {
              alive = false;
              break;
            }
            issue_S(t, static_cast<int>((kbase + jj) % C::kKS), sqm % SB);
            ++sqm;
            commit_me();
          }
          if (!alive) break;
          // the Q slot is free once this row block's last S MMA has run
          if ((!kTmaEpi || kOSep) && T <= SB) mma_commit(b_q_empty(qs));
          for (int j = 0; alive && j < T; ++j) {
            const int pb = pcm % SB;
            if (!mbar_wait(b_p_full(t, pb), (pcm / SB) & 1, abort_flag, wait_limit_ns)) {
              pp_give_up(misc, status, 7);
              alive = false;
              break;
            }
            ++pcm;
            const long long gv = kbase + j;  // V load number of tile j
            if (!mbar_wait(b_v_full(static_cast<int>(gv % C::kVS)), static_cast<int>(gv / C::kVS) & 1,
                           abort_flag, wait_limit_ns)) {
              pp_give_up(misc, status, 8);
              alive = false;
              break;
            }
            tc_fence_after();
            const uint32_t vb = dV0 + static_cast<uint32_t>(gv % C::kVS) * (C::kVBytes >> 4);
#pragma unroll
            for (int kk = 0; kk < BC / 16; ++kk)
              mma_ts(tO(t), tS(t, pb) + kk * 8, desc_join(vb + ((kk * 16 * 128) >> 4), kHi), idPV,
                     (j > 0 || kk > 0) ? 1u : 0u);
            if (j + SB < T) {  // S for key tile j + SB reuses the buffer P_t_j just left
              if (!wait_k(kbase + j + SB)) {
                alive = false;
                break;
              }
              issue_S(t, static_cast<int>((kbase + j + SB) % C::kKS), sqm % SB);
              ++sqm;
            }
            commit_me();
            if ((!kTmaEpi || kOSep) && j + SB + 1 == T) mma_commit(b_q_empty(qs));  // last S issued
          }
          kbase += it.Tmax;
        }
      } else
      for (long long k = 0, idx = item_idx(0); alive && idx < n_items; idx = item_idx(++k)) {
        const Item it = make_item<BC, CAUSAL, VARLEN>(idx, BH, n_pairs, n_rb, N, Hq, Hkv, group_major, cu_seqlens, total);
        if (VARLEN && it.T0 == 0) continue;  // a pair past the end of its sequence
        const int T[2] = {it.T0, it.T1};
        const int qs = items % C::kQS;
        dQ = sw128_desc_lo(sQ + qs * C::kQSlot, 16);
        if (!mbar_wait(b_q_full(qs), (items / C::kQS) & 1, abort_flag, wait_limit_ns)) {
          pp_give_up(misc, status, 5);
          break;
        }
        // prologue: S of the first SB key tiles, one commit per row block and tile
        for (int jj = 0; alive && jj < SB && jj < it.Tmax; ++jj) {
          if (!mbar_wait(b_k_full(kuse % C::kKS), (kuse / C::kKS) & 1, abort_flag, wait_limit_ns)) {
            pp_give_up(misc, status, 6);
            alive = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int t = 0; t < 2; ++t)
            if (jj < T[t]) {
              issue_S(t, kuse % C::kKS, sq[t] % SB);
              ++sq[t];
              commit(t);
            }
          ++kuse;
        }
        if (!alive) break;
        // the Q slot is free once the item's last S MMA has run
        if ((!kTmaEpi || kOSep) && it.Tmax <= SB) mma_commit(b_q_empty(qs));
        bool started[2] = {false, false};
        for (int j = 0; alive && j < it.Tmax; ++j) {
          bool v_used = false, k_next = false;
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            if (!alive || j >= T[t]) continue;
            const int pb = pc[t] % SB;
            if (!mbar_wait(b_p_full(t, pb), (pc[t] / SB) & 1, abort_flag, wait_limit_ns)) {
              pp_give_up(misc, status, 7);
              alive = false;
              continue;
            }
            ++pc[t];
            tc_fence_after();
            // every warp wrote its vote before arriving on p_full
            const int keep = SKIP ? decided_keep(t, dc[t] % kDR) : 1;
            ++dc[t];
            if (keep) {
              if (!v_used) {
                if (!mbar_wait(b_v_full(vuse % C::kVS), (vuse / C::kVS) & 1, abort_flag,
                               wait_limit_ns)) {
                  pp_give_up(misc, status, 8);
                  alive = false;
                  continue;
                }
                tc_fence_after();
                v_used = true;
              }
              const uint32_t vb = dV0 + (vuse % C::kVS) * (C::kVBytes >> 4);
#pragma unroll
              for (int kk = 0; kk < BC / 16; ++kk)
                mma_ts(tO(t), tS(t, pb) + kk * 8, desc_join(vb + ((kk * 16 * 128) >> 4), kHi), idPV,
                       (started[t] || kk > 0) ? 1u : 0u);
              started[t] = true;
            }
            // S for key tile j + SB reuses the buffer P_t_j just left
            if (j + SB < T[t]) {
              if (!k_next) {
                if (!mbar_wait(b_k_full(kuse % C::kKS), (kuse / C::kKS) & 1, abort_flag,
                               wait_limit_ns)) {
                  pp_give_up(misc, status, 9);
                  alive = false;
                  continue;
                }
                tc_fence_after();
                k_next = true;
              }
              issue_S(t, kuse % C::kKS, sq[t] % SB);
              ++sq[t];
            }
            commit(t);  // #(base_t + min(SB, T_t) + j): P*V_t_j and S_t_{j+SB}
          }
          if (k_next) ++kuse;
          if (v_used) ++vuse;
          if ((!kTmaEpi || kOSep) && j + SB + 1 == it.Tmax)
            mma_commit(b_q_empty(qs));  // last S MMAs issued
        }
        ++items;
      }
      // all issued MMAs must finish before TMEM is released
      mma_commit(b_mma_done(me));
      mbar_drain(b_mma_done(me), 0, wait_limit_ns);
    }
  } else {
    reg_inc<C::kSoftmaxRegs>();
    // -------------------------------------------------------- softmax warpgroups
    const int t = (warp - 4) >> 2;  // row block of the pair
    const int sw = warp & 3;        // TMEM sub-partition of this warp
    const int row = sw * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(sw * 32) << 16;
    const float NEG_INF = -__int_as_float(0x7f800000);
    int sc = 0, dcount = 0;
    int base = 0;    // this row block's commits in earlier items
    int items = 0;   // work items seen (the Q slot of item i is i % kQS)
    int leaves = 0;  // item-end synchronisations of this warpgroup
    // thread 0 of the warpgroup: the Q slot its last O store reads, and how
    // many arrivals on that slot's q_empty the store stands for
    int pend_slot = -1, pend_n = 0;
    auto release_pending = [&]() {
      if (kTmaEpi && pend_slot >= 0) {
        bulk_wait_read_all();
        if (!kOSep)
          for (int k = 0; k < pend_n; ++k) mbar_arrive(b_q_empty(pend_slot));
        pend_slot = -1;
      }
    };
    bool ok = true, failed = false;
    for (long long k = 0, idx = item_idx(0); ok && idx < n_items; idx = item_idx(++k)) {
      const Item it = make_item<BC, CAUSAL, VARLEN>(idx, BH, n_pairs, n_rb, N, Hq, Hkv, group_major, cu_seqlens, total);
      if (VARLEN && it.T0 == 0) continue;  // a pair past the end of its sequence: not a work item
      const int T = t == 0 ? it.T0 : it.T1;
      const int qs = items % C::kQS;
      ++items;
      if (T == 0) {  // this row block does not exist
        release_pending();
        continue;
      }
      const int pro = min(SB, T);
      const int rb = it.rb0 + t;
      const int q_idx = rb * kRows + row;
      const bool row_valid = q_idx < it.len;
      const size_t mask_base =
          skip_mask ? ((static_cast<size_t>(it.bh) * n_rb + rb) * n_tiles) : 0;
      float m_exact = NEG_INF, m_ref = NEG_INF, l_sum = 0.f;
      // log2-domain score scale; e4m3 scores carry the two per-head scales
      float sl2 = scale_log2;
      if constexpr (QK8)
        sl2 *= __ldg(q_scales + it.bh) *
               __ldg(k_scales + (it.bh / Hq) * Hkv + (it.bh % Hq) / (Hq / Hkv));
      for (int j = 0; j < T; ++j) {
        const int sb = sc % SB;  // S/P buffer of key tile j
        ++sc;
        bool waited = !failed && __all_sync(0xffffffffu, wait_cm(t, base + j));
        // raw scores stay in registers as fp32 bit patterns; the log2 scale is
        // folded into the max (positive scale) and into the exp FFMA below
        uint32_t u[BC];
        float mt = NEG_INF;
        if (waited) {
          tc_fence_after();
          tmem_ld_row<BC>(tS(t, sb) + lane_off, u);
          tmem_wait_ld();
          if constexpr (QKT == 2) {
            // int32 scores (|i| < 2^22 for 8-bit operands, d <= 128) become
            // the fp32 values 1.5 * 2^23 + i by one integer add to the bit
            // pattern of 1.5 * 2^23; the offset is taken out of the max below
            // and folded into the exponent's bias
#pragma unroll
            for (int c = 0; c < BC; ++c) u[c] += 0x4B400000u;
          }
          // last visible column of this row in tile j (-1: none); one integer
          // limit keeps the masking to a compare-select per column
          const int key0 = j * BC;
          int lim = min(BC - 1, it.len - 1 - key0);
          if (CAUSAL) lim = min(lim, q_idx - key0);
          if (!row_valid) lim = -1;
          if (lim < BC - 1) {
#pragma unroll
            for (int c = 0; c < BC; ++c) u[c] = (c > lim) ? 0xff800000u : u[c];
          }
          // row max: four independent chains of three-input maxima
          float m4[4] = {NEG_INF, NEG_INF, NEG_INF, NEG_INF};
#pragma unroll
          for (int c = 0; c < BC; c += 8)
#pragma unroll
            for (int k = 0; k < 4; ++k)
              m4[k] = fmax3(m4[k], __uint_as_float(u[c + 2 * k]), __uint_as_float(u[c + 2 * k + 1]));
          const float mraw = fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3]));
          // log2 units; -inf stays -inf; the int8 offset comes out exactly
          mt = (QKT == 2 ? mraw - kI2FOffset : mraw) * sl2;
        }
        // ---- skip test: every row of this row block must have mt < m - tau.
        // Each warp publishes its own verdict (all its rows pass, or not) and
        // arrives on the decision barrier.  A warp with a row that fails knows
        // at once that the tile is kept; only a warp whose rows all pass looks
        // at the other three verdicts, and stops at the first that fails.
        const int di = dcount % kDR;
        const int dnum = dcount;
        ++dcount;
        bool skip = false;
        if constexpr (SKIP) {  // with tau = inf every tile is kept and nobody reads votes
          const bool pass = waited &&
                            (!row_valid || (m_exact != NEG_INF && (mt == NEG_INF || mt < m_exact - tau_log2)));
          const bool warp_pass = __all_sync(0xffffffffu, pass) != 0;
          const bool warp_ok = waited;  // already the same in every lane (a warp vote)
          volatile int* vv = misc->vote[t][di];
          // every lane stores the same word (no divergent branch on the path
          // from S to P)
          vv[sw] = (dnum << 2) | (warp_ok ? 0 : 2) | (warp_pass ? 1 : 0);
          if (warp_pass) {
            int verdict = 0;  // 1 keep, 2 skip, 3 gave up
            if (lane == 0) {
              const uint64_t t0 = globaltimer_ns();
              for (uint32_t n = 0; verdict == 0; ++n) {
                int n_pass = 0;
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                  const int x = vv[w];
                  if ((x >> 2) == dnum) {
                    if (x & 1) ++n_pass;
                    else verdict = 1;
                  }
                }
                if (verdict == 0 && n_pass == 4) verdict = 2;
                if (verdict == 0 && (n & 15u) == 15u &&
                    (*abort_flag || globaltimer_ns() - t0 > wait_limit_ns))
                  verdict = 3;
                if (verdict == 0 && n >= 2) __nanosleep(64);  // leave the issue slots to the others
              }
            }
            verdict = __shfl_sync(0xffffffffu, verdict, 0);
            if (verdict == 3) waited = false;
            skip = verdict == 2;
          }
        }
        if (!waited) {
          // The warps of this row block run out the item and leave together
          // at the item-end synchronisation below.
          if (!failed) pp_give_up(misc, status, 10);
          failed = true;
          continue;
        }
        m_exact = fmaxf(m_exact, mt);
        if (row == 0 && skip_mask) skip_mask[mask_base + j] = skip ? 1 : 0;
        if (skip) {
          __syncwarp();
          if (lane == 0) mbar_arrive(b_p_full(t, sb));
          if (j == 0) release_pending();
          continue;
        }
        // ---- kept tile: lazy reference max, P, then O rescale
        const float m_cand = fmaxf(m_ref, mt);
        const bool moved = row_valid && (m_cand > m_ref + kRescale);
        float alpha = 1.f;
        if (moved) {
          alpha = ex2(m_ref - m_cand);
          m_ref = m_cand;
        }
        // P = 2^(s*scale - m_ref): one packed FFMA per pair, two ex2, one
        // pack to bf16 for the P*V MMA.  The row sum adds the bf16-rounded
        // pair that the P*V MMA multiplies (one packed add, four independent
        // chains), so numerator and denominator see the same weights and the
        // rounding of a dominant weight cancels in O / l.
        // invalid rows: all scores -inf -> P = 0; int8 scores carry the
        // offset 1.5 * 2^23, taken out here
        const float neg_m = (row_valid ? -m_ref : 0.f) - (QKT == 2 ? kI2FOffset * sl2 : 0.f);
        const float2 sc2 = make_float2(sl2, sl2);
        const float2 nm2 = make_float2(neg_m, neg_m);
        float2 rs2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                         make_float2(0.f, 0.f)};  // four independent add chains
#pragma unroll
        for (int c0 = 0; c0 < BC; c0 += 32) {
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const float2 x = __ffma2_rn(
                make_float2(__uint_as_float(u[c0 + 2 * c]), __uint_as_float(u[c0 + 2 * c + 1])), sc2,
                nm2);
            // pairs in kPolyPairs take 2^x on the FMA pipes, the rest on MUFU
            const uint32_t w = ((kPolyPairs >> c) & 1u) ? exp2_poly_bf16x2(x)
                                                        : pack_bf16x2(ex2(x.x), ex2(x.y));
            rs2[c & 3] = __fadd2_rn(rs2[c & 3], make_float2(__uint_as_float(w << 16),
                                                            __uint_as_float(w & 0xffff0000u)));
            pk[c] = w;
          }
          tmem_st16(tS(t, sb) + lane_off + c0 / 2, pk);
        }
        const float2 rsa = __fadd2_rn(__fadd2_rn(rs2[0], rs2[1]), __fadd2_rn(rs2[2], rs2[3]));
        l_sum = l_sum * alpha + (rsa.x + rsa.y);
        // O rescale (after the P store, so the scores are no longer live).
        // P*V of tile j-1 must have finished: commit #(base + pro + j - 1).
        // With one S buffer that is the commit S_j already waited for.
        if (j > 0 && __any_sync(0xffffffffu, moved)) {
          if (SB > 1 && !__all_sync(0xffffffffu, wait_cm(t, base + pro + j - 1))) {
            pp_give_up(misc, status, 12);
            failed = true;  // acted on at the next vote, or just below
          }
          if (!failed) {
            tc_fence_after();
            const float a = moved ? alpha : 1.f;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
              uint32_t r[32];
              tmem_ld32(tO(t) + lane_off + c0, r);
              tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < 32; ++c) r[c] = __float_as_uint(__uint_as_float(r[c]) * a);
              tmem_st32(tO(t) + lane_off + c0, r);
            }
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(b_p_full(t, sb));
        // the previous item's O store has had a tile's time to read its Q slot
        if (j == 0) release_pending();
      }
      // ---- epilogue: O / l -> bf16 -> global; unvisited tiles marked 2
      if (skip_mask)
        for (int j = T + row; j < n_tiles; j += 128) skip_mask[mask_base + j] = 2;
      // P*V of the last tile finished: commit #(base + pro + T - 1).  A give-up
      // (recorded by any warp during the item) or a failed wait is combined
      // over the four warps, which then go on, or leave, together.
      bool done = !failed && __all_sync(0xffffffffu, wait_cm(t, base + pro + T - 1));
      base += pro + T;
      {
        volatile int* lv = misc->leave[t][leaves & 1];
        ++leaves;
        if (lane == 0) lv[sw] = done ? 0 : 1;
        named_bar(1 + t, 128);
#pragma unroll
        for (int w = 0; w < 4; ++w)
          if (lv[w]) done = false;
      }
      if (!done) {
        if (!failed) pp_give_up(misc, status, 11);
        ok = false;
        break;
      }
      tc_fence_after();
      const float inv_l = row_valid ? 1.f / l_sum : 0.f;
      const bool tma_store = kTmaEpi && (!VARLEN || (rb + 1) * kRows <= it.len);
      if (tma_store) {
        // Stage O (bf16) in this row block's Q tile, which no MMA reads any
        // more (its last S MMA completed before the last P*V), in the TMA
        // layout (64-column panels, 128-byte swizzle), then one thread stores
        // the tile; rows past N are clipped by the store.
        const uint32_t stage =
            kOSep ? sbase + C::kOffO + t * C::kOTile : sQ + qs * C::kQSlot + t * C::kQTile;
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t r[32];
          tmem_ld32(tO(t) + lane_off + c0, r);
          tmem_wait_ld();
          uint32_t w[16];
#pragma unroll
          for (int c = 0; c < 16; ++c)
            w[c] = pack_bf16x2(__uint_as_float(r[2 * c]) * inv_l, __uint_as_float(r[2 * c + 1]) * inv_l);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int lc = c0 / 8 + q;  // 16-byte chunk of the row
            const uint32_t a = stage + (lc >> 3) * C::kQPanel + row * 128 + (((lc & 7) ^ (row & 7)) << 4);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(w[4 * q]),
                         "r"(w[4 * q + 1]), "r"(w[4 * q + 2]), "r"(w[4 * q + 3])
                         : "memory");
          }
        }
        fence_proxy_async_smem();  // the generic-proxy writes, before the async-proxy store
        named_bar(1 + t, 128);
        if (row == 0) {
          release_pending();  // at most one store in flight per warpgroup
#pragma unroll
          for (int p = 0; p < C::kVPanels; ++p) {
            if constexpr (VARLEN)  // O as [tokens, Hq, d]
              tma_store_3d(&tmO, stage + p * C::kQPanel, p * 64, it.bh % Hq, it.tok0 + rb * kRows);
            else
              tma_store_3d(&tmO, stage + p * C::kQPanel, p * 64, rb * kRows, it.bh);
          }
          bulk_commit_group();
          pend_slot = qs;
          pend_n = (t == 0 && it.T1 == 0) ? 2 : 1;  // row block 1 absent: arrive for it too
        }
      } else {
        __nv_bfloat16* orow =
            VARLEN ? O + (static_cast<size_t>(it.tok0 + (row_valid ? q_idx : 0)) * Hq + it.bh % Hq) * D
                   : O + (static_cast<size_t>(it.bh) * N + (row_valid ? q_idx : 0)) * D;
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t r[32];
          tmem_ld32(tO(t) + lane_off + c0, r);
          tmem_wait_ld();
          if (row_valid) {
            uint32_t w[16];
#pragma unroll
            for (int c = 0; c < 16; ++c)
              w[c] = pack_bf16x2(__uint_as_float(r[2 * c]) * inv_l, __uint_as_float(r[2 * c + 1]) * inv_l);
            uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
            for (int q = 0; q < 4; ++q) dst[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
          }
        }
        if (kTmaEpi && row == 0) {  // no store reads the Q slot: hand it back like one
          release_pending();
          pend_slot = qs;
          pend_n = (t == 0 && it.T1 == 0) ? 2 : 1;
        }
      }
      // O_t may be overwritten by the next item's first P*V only after this
      // warpgroup signals that item's first P: ordering comes from p_full.
      tc_fence_before();
    }
    // no store may still be reading shared memory, or writing O, at exit
    release_pending();
    if (kTmaEpi && row == 0) bulk_wait_all();
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

PFN_cuTensorMapEncodeTiled_v12000 pp_encoder() {
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

bool pp_map(CUtensorMap* m, const void* base, int BH, int rows, int D, int box_rows) {
  auto enc = pp_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(rows) * D * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [BH, N, D] e4m3 (one byte per element), d fastest; box = 128 columns (one
// 128-byte swizzle row) x box_rows rows.
bool pp_map_e4m3(CUtensorMap* m, const void* base, int BH, int N, int D, int box_rows) {
  auto enc = pp_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(N) * D};
  cuuint32_t box[3] = {128, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [tokens, H, D] bf16 (variable-length batches), d fastest; box = 64 columns
// x 1 head x box_rows tokens, so the tile in shared memory is laid out as in
// pp_map.  Tokens past the end of the tensor read as zeros.
bool pp_map_thd(CUtensorMap* m, const void* base, int H, int tokens, int D, int box_rows) {
  auto enc = pp_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(tokens)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(H) * D * 2};
  cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// [BH, rows, D] bf16, d fastest: 64-column boxes of box_rows rows, 128-byte
// swizzle (shared with the column-split prefill kernel).
bool tma_map_bhnd(CUtensorMap* m, const void* base, int BH, int rows, int D, int box_rows) {
  return pp_map(m, base, BH, rows, D, box_rows);
}

namespace {

template <int D, int BC, bool CAUSAL, bool VARLEN, int QKT, bool SKIP>
int pp_launch_t(const PrefillLaunch& a) {
  constexpr bool QK8 = QKT != 0;
  using C = PPCfg<D, BC, QK8>;
  auto kern = prefill_pp_kernel<D, BC, CAUSAL, VARLEN, QKT, SKIP>;
  static uint64_t ready = 0;  // one bit per device: attributes set and checked
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return ATTN_ERR_CUDA;
  static int sm_count[64];
  if (!(ready >> dev & 1)) {
    // The register split (setmaxnreg) assumes exactly kPPRegs registers per
    // thread at launch; anything else could leave setmaxnreg.inc waiting.
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return ATTN_ERR_CUDA;
    if (fa.numRegs != kPPRegs) return ATTN_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
        cudaSuccess)
      return ATTN_ERR_CUDA;
    if (cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return ATTN_ERR_CUDA;
    ready |= uint64_t(1) << dev;
  }
  CUtensorMap mq, mk, mv, mo;
  if (VARLEN) {
    if (!pp_map_thd(&mq, a.Q, a.Hq, a.total, D, kRows) ||
        !pp_map_thd(&mk, a.K, a.Hkv, a.total, D, BC) || !pp_map_thd(&mv, a.V, a.Hkv, a.total, D, BC))
      return ATTN_ERR_CUDA;
    if (!pp_map_thd(&mo, a.O, a.Hq, a.total, D, kRows)) return ATTN_ERR_CUDA;
    if (a.skip_mask) {  // row blocks past a sequence's end are never visited
      const size_t n = static_cast<size_t>(a.B) * a.Hq * ((a.N + kRows - 1) / kRows) *
                       ((a.N + BC - 1) / BC);
      if (cudaMemsetAsync(a.skip_mask, 2, n, a.stream) != cudaSuccess) return ATTN_ERR_CUDA;
    }
  } else if (QK8) {
    if (!pp_map_e4m3(&mq, a.Q, a.B * a.Hq, a.N, D, kRows) ||
        !pp_map_e4m3(&mk, a.K, a.B * a.Hkv, a.N, D, BC) ||
        !pp_map(&mv, a.V, a.B * a.Hkv, a.N, D, BC))
      return ATTN_ERR_CUDA;
    if (!C::kOSep) mo = mv;  // unused: O is stored row by row
    else if (!pp_map(&mo, a.O, a.B * a.Hq, a.N, D, kRows)) return ATTN_ERR_CUDA;
  } else if (!pp_map(&mq, a.Q, a.B * a.Hq, a.N, D, kRows) ||
             !pp_map(&mk, a.K, a.B * a.Hkv, a.N, D, BC) ||
             !pp_map(&mv, a.V, a.B * a.Hkv, a.N, D, BC) ||
             !pp_map(&mo, a.O, a.B * a.Hq, a.N, D, kRows)) {
    return ATTN_ERR_CUDA;
  }
  const long long n_rb = (a.N + kRows - 1) / kRows;
  const long long n_items = static_cast<long long>(a.B) * a.Hq * ((n_rb + 1) / 2);
  const int grid = static_cast<int>(n_items < sm_count[dev] ? n_items : sm_count[dev]);
  kern<<<grid, kPPThreads, C::kSmemBytes, a.stream>>>(
      mq, mk, mv, mo, static_cast<__nv_bfloat16*>(a.O), a.skip_mask, a.status, a.B, a.Hq, a.Hkv, a.N,
      a.scale_log2, a.tau_log2, a.wait_limit_ns, a.cu_seqlens, a.total, a.q_scales, a.k_scales);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <int D, int BC, bool CAUSAL, bool VARLEN, int QKT>
int pp_launch(const PrefillLaunch& a) {
  return a.tau_is_inf ? pp_launch_t<D, BC, CAUSAL, VARLEN, QKT, false>(a)
                      : pp_launch_t<D, BC, CAUSAL, VARLEN, QKT, true>(a);
}

template <int D, int BC>
int pp_launch_c(const PrefillLaunch& a) {
  if (a.cu_seqlens)
    return a.causal ? pp_launch<D, BC, true, true, 0>(a) : pp_launch<D, BC, false, true, 0>(a);
  return a.causal ? pp_launch<D, BC, true, false, 0>(a) : pp_launch<D, BC, false, false, 0>(a);
}

}  // namespace

int launch_prefill_pp(const PrefillLaunch& a) {
  if (a.Br != 128) return ATTN_ERR_INVALID_ARG;
  if (a.q_scales) {  // 8-bit Q and K: d = 128, fixed-length batches
    if (a.d != 128 || a.cu_seqlens) return ATTN_ERR_INVALID_ARG;
    if (a.qk_format == 1) {
      if (a.Bc == 64)
        return a.causal ? pp_launch<128, 64, true, false, 1>(a) : pp_launch<128, 64, false, false, 1>(a);
      return a.causal ? pp_launch<128, 128, true, false, 1>(a) : pp_launch<128, 128, false, false, 1>(a);
    }
    if (a.qk_format == 2) {
      if (a.Bc == 64)
        return a.causal ? pp_launch<128, 64, true, false, 2>(a) : pp_launch<128, 64, false, false, 2>(a);
      return a.causal ? pp_launch<128, 128, true, false, 2>(a) : pp_launch<128, 128, false, false, 2>(a);
    }
    return ATTN_ERR_INVALID_ARG;
  }
  // d = Bc = 128, fixed length: the column-split kernel (three S buffers
  // beside one O accumulator; measured faster than two row blocks per CTA,
  // whose one S buffer per row block serialises S, softmax and P*V).  Bc = 64
  // keeps two row blocks per CTA with two S buffers each, measured faster.
  if (a.d == 128 && a.Bc == 128 && !a.cu_seqlens) return launch_prefill_split(a);
  if (a.d == 128) return a.Bc == 64 ? pp_launch_c<128, 64>(a) : pp_launch_c<128, 128>(a);
  if (a.d == 64) return a.Bc == 64 ? pp_launch_c<64, 64>(a) : pp_launch_c<64, 128>(a);
  return ATTN_ERR_INVALID_ARG;
}

}  // namespace bss
