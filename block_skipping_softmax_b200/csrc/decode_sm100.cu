// Skip Softmax decode attention for sm_100a (B200): split-KV, grouped-query.
//
// Method: "Accelerating Long-Context Inference with Skip Softmax in NVIDIA
// TensorRT-LLM" (Key Points; Detailed Analysis) -- a block of keys whose
// local maximum score lies more than tau below the running maximum of every
// query row is skipped, which saves its exponentials and its value reads
// (the page credits the method with lower memory-bandwidth pressure).  In
// decode the rows of the test are the g = Hq/Hkv query heads that share one
// KV head, because they share the V tile that a skip avoids reading.
//
// Work split: CTA (split, kv head, batch) streams its split's 64-key tiles.
// Decode is bound by HBM reads of K and V; a g-row GEMV does not fill an MMA,
// so the arithmetic runs on the FMA pipes and the design goal is the fewest
// issued instructions per byte, so that the memory system stays the limit:
//
//  * Tiles arrive by TMA as 64-column panels with the 128-byte swizzle (16 KB
//    per d=128 tile), K three tiles ahead of the compute; a V tile is
//    requested only once its tile is known to be kept and is consumed two
//    iterations later.  The swizzle lets a group of eight lanes read eight
//    different keys (or eight chunks of one key) without bank conflicts, so
//    each lane can hold several 16-byte chunks of a key row and the cross-lane
//    reduction of a score shrinks to a few butterfly steps.
//  * Scores: kP lanes share a key, each with kCPL chunks of q and k in fp32,
//    packed FMAs; the butterfly transposes so that a lane ends up with the
//    score of one (key, query row).  The 1/sqrt(d) and log2(e) factors are
//    folded into q.
//  * One CTA barrier per tile.  After it every warp takes the same skip
//    decision lane-parallel (lane = one (warp, row) maximum, a 3-step max
//    butterfly, one vote), so no warp waits on a serial decision phase.
//  * A lazy reference max per row: probabilities are taken relative to a
//    value that is moved up only when the running max exceeds it by more
//    than 2^8, so the partial sums are rescaled rarely.  The skip test itself
//    always uses the exact running max.
//  * P*V: a thread owns one 16-byte chunk of d for all g rows and a fixed
//    subset of the tile's keys; the sums over key subsets are combined once
//    at the end of the split.
//
// Output per split: normalised partial o (fp32) and its log2-sum-exp; a second
// kernel merges the splits exactly.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

#include "kernels.cuh"
#include "ptx.cuh"

namespace bss {

namespace {

constexpr int kWarps = 8;
constexpr int kDecThreads = kWarps * 32;
constexpr int kKStages = 3;  // K tiles in flight ahead of the compute
constexpr int kLag = 2;      // a kept tile's P*V runs kLag iterations after its test
constexpr int kVStages = kLag + 1;
constexpr int kPRing = kLag + 1;
constexpr float kRefSlack = 8.f;  // log2 units: probabilities stay below 2^8
constexpr int kPageChunk = 512;   // paged cache: tiles whose pages are staged at a time
constexpr int kPageSlots = 2 * kPageChunk;

template <int D, int G>
struct DecCfg {
  static constexpr int kPanels = D / 64;                 // 64-column panels per key row
  static constexpr int kPanelBytes = kDecodeTile * 128;  // 64 keys x 128 B
  static constexpr int kTileBytes = kPanels * kPanelBytes;
  static constexpr int kChunks = D / 8;  // 16-byte chunks per key row
  // score phase: kP lanes share a key, each holding kCPL chunks of q (at most
  // 64 fp32 values of q per lane)
  static constexpr int kCPL = (kChunks / 4 < 8 / G) ? kChunks / 4 : 8 / G;
  static constexpr int kP = kChunks / kCPL;
  static constexpr int kKPI = 32 / kP;                 // keys per warp instruction
  static constexpr int kKeysPerWarp = kDecodeTile / kWarps;
  static constexpr int kSIters = kKeysPerWarp / kKPI;  // score iterations per tile
  static constexpr bool kKeyMajor = kP >= 8;           // lane = key * kP + qd, else qd * kKPI + key
  static constexpr int kDup = kP / G;                  // lanes holding the same (key, row) score
  // P*V phase: kChunks lanes per key, kGroups disjoint key subsets
  static constexpr int kGroups = kDecThreads / kChunks;
  static constexpr int kVKeys = kDecodeTile / kGroups;
  // shared memory (offsets from a 1024-byte aligned base)
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kKStages * kTileBytes;
  static constexpr int kOffP = kOffV + kVStages * kTileBytes;          // float [ring][64][G]
  static constexpr int kOffR = kOffP + kPRing * kDecodeTile * G * 4;   // float [ring][8] ref max
  static constexpr int kOffF = kOffR + kPRing * 8 * 4;                 // int [ring] rescale flag
  static constexpr int kOffW = kOffF + 16;                             // float [2][warps][G]
  static constexpr int kOffL = kOffW + 2 * kWarps * G * 4;             // float [warps][G]
  static constexpr int kOffMisc = kOffL + kWarps * G * 4;
  static constexpr int kOffBar = kOffMisc + 16;
  static constexpr int kSmemUsed = kOffBar + 8 * (kKStages + kVStages + 1);  // + sink-seed tile
  static constexpr int kSmemBytes = kSmemUsed + 1024;  // room to align the base
  // paged cache only: int [kPageSlots] pages of the split's tiles
  static constexpr int kOffTab = (kSmemUsed + 15) / 16 * 16;
  static constexpr int kSmemBytesPaged = kOffTab + kPageSlots * 4 + 1024;
  static_assert(G <= kP, "a lane ends the butterfly with one row");
  static_assert(kSIters >= 1 && kKPI * kSIters == kKeysPerWarp, "score lane layout");
  static_assert(kKeyMajor || kKPI == 8, "qd-major lanes need eight keys per instruction");
  static_assert(kChunks >= 8 && kGroups * kVKeys == kDecodeTile, "P*V lane layout");
  static_assert(kWarps * G * D * 4 <= kKStages * kTileBytes, "reduction scratch");
  static_assert(G <= 8 && kOffP % 16 == 0, "ring layout");
};

constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x / 2); }

// byte offset of 16-byte chunk `lc` of key row `k` in a tile of swizzled panels
template <int D>
__device__ __forceinline__ uint32_t chunk_off(int k, int lc) {
  return static_cast<uint32_t>((lc >> 3) * (kDecodeTile * 128) + k * 128 +
                               (((lc & 7) ^ (k & 7)) << 4));
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4 u, float2 (&f)[4]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int e = 0; e < 4; ++e)
    f[e] = make_float2(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xffff0000u));
}

template <int G>
__device__ __forceinline__ void load_row_floats(const float* p, float (&v)[G]) {
  if constexpr (G % 4 == 0) {
#pragma unroll
    for (int i = 0; i < G; i += 4) {
      const float4 x = *reinterpret_cast<const float4*>(p + i);
      v[i] = x.x; v[i + 1] = x.y; v[i + 2] = x.z; v[i + 3] = x.w;
    }
  } else if constexpr (G == 2) {
    const float2 x = *reinterpret_cast<const float2*>(p);
    v[0] = x.x; v[1] = x.y;
  } else {
    v[0] = p[0];
  }
}

}  // namespace

// SKIP: tau is finite, so the kernel takes the skip test; with tau = inf it
// holds no trace of it.
template <int D, int G, int RULE, bool PAGED, bool SKIP>
__global__ void __launch_bounds__(kDecThreads, (G <= 4) ? 2 : 1)
    decode_partial_kernel(const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV,
                          const __nv_bfloat16* __restrict__ q, float* __restrict__ o_part,
                          float* __restrict__ lse_part, uint8_t* __restrict__ skip_mask,
                          int* __restrict__ status, int Hq, int Hkv, int L, int split_len,
                          int n_splits, float scale_log2, float tau_log2,
                          unsigned long long wait_limit_ns, int withhold_v,
                          const int* __restrict__ block_table, const int* __restrict__ seq_lens,
                          int max_pages) {
  using C = DecCfg<D, G>;
  constexpr unsigned FULL = 0xffffffffu;
  constexpr int kLog2P = ilog2(C::kP);
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;  // the swizzle pattern repeats every 1024 B
  uint8_t* smem = smem_raw + (sbase - raw);
  float* p_ring = reinterpret_cast<float*>(smem + C::kOffP);
  float* ref_ring = reinterpret_cast<float*>(smem + C::kOffR);
  int* flag_ring = reinterpret_cast<int*>(smem + C::kOffF);
  float* wmax = reinterpret_cast<float*>(smem + C::kOffW);
  float* wl = reinterpret_cast<float*>(smem + C::kOffL);
  // Give-ups are made CTA-uniform with __syncthreads_or, so no role ever
  // needs to be told to stop early: this flag stays 0.
  volatile int* never = reinterpret_cast<volatile int*>(smem + C::kOffMisc);
  const uint32_t bar0 = sbase + C::kOffBar;
  auto b_k_full = [&](int s) { return bar0 + 8u * s; };
  auto b_v_full = [&](int s) { return bar0 + 8u * (kKStages + s); };
  const uint32_t b_seed = bar0 + 8u * (kKStages + kVStages);
  // the rule variant is a template argument, so the default rule carries no trace of the others
  constexpr bool per_head = (RULE & ATTN_DECODE_RULE_PER_HEAD) != 0;
  constexpr bool seeded = (RULE & ATTN_DECODE_RULE_SINK_SEED) != 0;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int split = blockIdx.x;
  const int kv = blockIdx.y;
  const int b = blockIdx.z;
  const int bh = b * Hkv + kv;
  // Paged KV cache: L is the longest sequence; this one has Lb keys, clamped
  // to what its row of the block table can address.
  int Lb = L;
  if constexpr (PAGED) Lb = max(0, min(min(seq_lens[b], L), max_pages * kDecodeTile));
  const int n_tiles_all = (L + kDecodeTile - 1) / kDecodeTile;  // length of a mask row
  const int n_tiles_b = (Lb + kDecodeTile - 1) / kDecodeTile;
  const int tps = split_len / kDecodeTile;
  const int t_begin = split * tps;
  const int t_end = min(n_tiles_b, t_begin + tps);
  const int nt = t_end - t_begin;
  const float NEG_INF = -__int_as_float(0x7f800000);

  if constexpr (PAGED) {
    // tiles of this split past the end of the sequence are not visited
    if (skip_mask) {
      const int rows = per_head ? G : 1;
      for (int idx = tid; idx < rows * tps; idx += kDecThreads) {
        const int t = t_begin + idx % tps, r = idx / tps;
        if (t >= n_tiles_b && t < n_tiles_all) {
          const size_t mrow = per_head ? static_cast<size_t>(b) * Hq + kv * G + r : bh;
          skip_mask[mrow * n_tiles_all + t] = 2;
        }
      }
    }
    if (nt <= 0) {  // the whole split lies past the end: zero weight in the merge
      for (int idx = tid; idx < G * D; idx += kDecThreads) {
        const size_t row = static_cast<size_t>(b) * Hq + kv * G + idx / D;
        o_part[(row * n_splits + split) * D + idx % D] = 0.f;
      }
      if (tid < G) lse_part[(static_cast<size_t>(b) * Hq + kv * G + tid) * n_splits + split] = NEG_INF;
      return;
    }
  }

  // Paged: the pages of the split's tiles are staged in shared memory (tile
  // k of the split in slot k % kPageSlots) by all threads, kPageChunk at a
  // time and a whole chunk before any copy needs them, so the thread that
  // issues the copies never reads the block table itself: a table read on
  // that path (an L2 round trip per tile under full HBM load) held every
  // warp at the next barrier.  Entries past the split's last tile are never
  // read (t_end <= the tiles the table row addresses).
  int* pg_tab = reinterpret_cast<int*>(smem + C::kOffTab);
  auto stage_pages = [&](int k0) {  // tiles k0 .. k0 + kPageChunk - 1 (those < nt)
    const int* bt_row = block_table + static_cast<size_t>(b) * max_pages + t_begin;
    const int k1 = min(nt, k0 + kPageChunk);
    for (int k = k0 + tid; k < k1; k += kDecThreads) pg_tab[k % kPageSlots] = bt_row[k];
  };

  // one tile = kPanels TMA boxes of 64 columns x 64 keys; rows past L read as
  // zeros.  Paged: tile t of this sequence is page block_table[b][t], whose
  // 64 keys of KV head kv are row (page * Hkv + kv) of the page pool; the
  // caller passes the page (unused for the contiguous cache).
  auto issue = [&](uint32_t dst, const CUtensorMap* map, uint32_t bar, int t, int page) {
    mbar_arrive_expect_tx(bar, C::kTileBytes);
    int c1 = t * kDecodeTile, c2 = bh;
    if constexpr (PAGED) {
      c1 = 0;
      c2 = page * Hkv + kv;
    }
#pragma unroll
    for (int p = 0; p < C::kPanels; ++p)
      tma_load_3d(dst + p * C::kPanelBytes, map, bar, p * 64, c1, c2);
  };
  if constexpr (PAGED) {  // chunks 0 and 1, published by the barrier below
    stage_pages(0);
    stage_pages(kPageChunk);
  }

  if (tid == 0) {
    for (int s = 0; s < kKStages; ++s) mbar_init(b_k_full(s), 1);
    for (int s = 0; s < kVStages; ++s) mbar_init(b_v_full(s), 1);
    mbar_init(b_seed, 1);
    *never = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  __syncthreads();
  int k_issued = 0, v_issued = 0;
  if (tid == 0) {
    for (int i = 0; i < kKStages && i < nt; ++i) {
      issue(sbase + C::kOffK + i * C::kTileBytes, &tmK, b_k_full(i), t_begin + i,
            PAGED ? pg_tab[i] : 0);
      ++k_issued;
    }
  }

  // score-phase roles: lane holds chunks lc = j*kP + qd of key kl; after the
  // butterfly it holds the score of (key, row_q)
  const int qd = C::kKeyMajor ? (lane % C::kP) : (lane / C::kKPI);
  const int kl = C::kKeyMajor ? (lane / C::kP) : (lane % C::kKPI);
  const int row_q = qd / C::kDup;
  const bool leader = (qd % C::kDup) == 0;
  // P*V roles: chunk ch of d, keys kg + kGroups*e
  const int ch = lane % C::kChunks;
  const int kg = warp * (32 / C::kChunks) + lane / C::kChunks;
  // decision roles: lane < n_dec holds the maximum of (warp lane/G, row lane%G)
  constexpr int n_dec = (8 * G < 32) ? 8 * G : 32;

  float2 qf[G][C::kCPL][4];
#pragma unroll
  for (int r = 0; r < G; ++r) {
#pragma unroll
    for (int j = 0; j < C::kCPL; ++j) {
      const uint4 u = *reinterpret_cast<const uint4*>(
          q + (static_cast<size_t>(b) * Hq + kv * G + r) * D + (j * C::kP + qd) * 8);
      bf16x8_to_f32(u, qf[r][j]);
#pragma unroll
      for (int e = 0; e < 4; ++e)
        qf[r][j][e] = __fmul2_rn(qf[r][j][e], make_float2(scale_log2, scale_log2));
    }
  }

  float m_exact = NEG_INF;  // decision lanes: exact running max of row lane % G (log2 units)
  float m_ref = NEG_INF;    // decision lanes: reference max of that row
  float lsum = 0.f;         // leader score lanes: sum of p for row row_q over this lane's keys
  float2 acc[G][4];         // P*V threads: rows x 8 columns of chunk ch
  float m_acc[G];           // P*V threads: reference max the sums in acc are relative to
#pragma unroll
  for (int r = 0; r < G; ++r) {
    m_acc[r] = NEG_INF;
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[r][e] = make_float2(0.f, 0.f);
  }
  uint32_t kept_bits = 0;  // bit k: tile i - k was kept
  int pv_count = 0;        // V tiles consumed
  bool ok = true;          // this thread's waits so far succeeded

  // Scores of one K tile in shared memory (keys >= key_lim are past L and
  // read as -inf) into sv; returns this warp's maximum for row_q.
  auto tile_scores = [&](const uint8_t* kt, int key_lim, float (&sv)[C::kSIters]) -> float {
    float wm = NEG_INF;
#pragma unroll
    for (int it = 0; it < C::kSIters; ++it) {
      const int key = warp * C::kKeysPerWarp + it * C::kKPI + kl;
      float2 s2[G];
#pragma unroll
      for (int r = 0; r < G; ++r) s2[r] = make_float2(0.f, 0.f);
#pragma unroll
      for (int j = 0; j < C::kCPL; ++j) {
        const uint4 u = *reinterpret_cast<const uint4*>(kt + chunk_off<D>(key, j * C::kP + qd));
        float2 kf[4];
        bf16x8_to_f32(u, kf);
#pragma unroll
        for (int r = 0; r < G; ++r)
#pragma unroll
          for (int e = 0; e < 4; ++e) s2[r] = __ffma2_rn(qf[r][j][e], kf[e], s2[r]);
      }
      float v[G];
#pragma unroll
      for (int r = 0; r < G; ++r) v[r] = s2[r].x + s2[r].y;
      // butterfly over the kP lanes of this key, highest qd bit first: the
      // first log2(G) steps each keep half of the rows (the lanes with the
      // bit set keep the upper half), the rest are plain sums
#pragma unroll
      for (int s = 0; s < kLog2P; ++s) {
        const int qbit = kLog2P - 1 - s;
        const int o = C::kKeyMajor ? (1 << qbit) : (C::kKPI << qbit);
        const int n = G >> s;
        if (n > 1) {
          const int hh = n / 2;
          const bool upper = ((qd >> qbit) & 1) != 0;
#pragma unroll
          for (int r = 0; r < hh; ++r) {
            const float send = upper ? v[r] : v[r + hh];
            const float keep = upper ? v[r + hh] : v[r];
            v[r] = keep + __shfl_xor_sync(FULL, send, o);
          }
        } else {
          v[0] += __shfl_xor_sync(FULL, v[0], o);
        }
      }
      sv[it] = key < key_lim ? v[0] : NEG_INF;
      wm = fmaxf(wm, sv[it]);
    }
    // max over the warp's keys for row_q
    if constexpr (C::kKeyMajor) {
#pragma unroll
      for (int o = C::kP; o < 32; o <<= 1) wm = fmaxf(wm, __shfl_xor_sync(FULL, wm, o));
    } else {
#pragma unroll
      for (int o = 1; o < C::kKPI; o <<= 1) wm = fmaxf(wm, __shfl_xor_sync(FULL, wm, o));
    }
    return wm;
  };

  // Sink seed: the running max of a split other than the first starts at the
  // rows' maximum over the sequence's first key tile (where attention sinks
  // sit) instead of -inf.  The tile goes to V slot 0, free until the first
  // V copy, which is issued only after the first decision.
  bool seed_issued = false;
  if (seeded && t_begin > 0) {
    if (tid == 0) {
      issue(sbase + C::kOffV, &tmK, b_seed, 0,
            PAGED ? block_table[static_cast<size_t>(b) * max_pages] : 0);
      seed_issued = true;
    }
    const bool got = mbar_wait(b_seed, 0, never, wait_limit_ns);
    ok = ok && got;
    float sv0[C::kSIters];
    const float wm0 = tile_scores(smem + C::kOffV, Lb, sv0);
    if (kl == 0 && leader) wmax[(kWarps + warp) * G + row_q] = wm0;  // buffer 1; tile 0 uses buffer 0
    __syncthreads();
    const float* wb = wmax + kWarps * G;
    float mt = lane < n_dec ? wb[lane] : NEG_INF;
    if constexpr (G == 8) mt = fmaxf(mt, wb[lane + 32]);
#pragma unroll
    for (int o = G; o < n_dec; o <<= 1) mt = fmaxf(mt, __shfl_xor_sync(FULL, mt, o));
    m_exact = lane < n_dec ? mt : NEG_INF;
  }

  for (int i = 0; i < nt + kLag; ++i) {
    // ---------------- A: scores of tile i and the per-warp row maxima
    float sv[C::kSIters];
    if (i < nt) {
      const int ks = i % kKStages;
      const bool got = mbar_wait(b_k_full(ks), (i / kKStages) & 1, never, wait_limit_ns);
      ok = ok && got;  // on a give-up the scores are garbage and dropped at the barrier
      const uint8_t* kt = smem + C::kOffK + ks * C::kTileBytes;
      const int key_lim = Lb - (t_begin + i) * kDecodeTile;  // keys >= key_lim are past the end
      const float wm = tile_scores(kt, key_lim, sv);
      if (kl == 0 && leader) wmax[((i & 1) * kWarps + warp) * G + row_q] = wm;
    }
    if (__syncthreads_or(!ok)) {  // the single per-tile barrier; also a uniform give-up
      ok = false;
      break;
    }
    // ---------------- B: decision for tile i, taken identically by every warp
    bool keep_i = false;
    if (i < nt) {
      // paged: the pages of this iteration's copies (V of tile i, K of tile
      // i + kKStages) are read here, beside the row maxima, by every thread,
      // so the issuing thread does not wait for them after the decision
      // (when the other warps' P*V loads fill the shared-memory pipe, and
      // every warp waits for the issuing one at the next barrier)
      int pg_v = 0, pg_k = 0;
      if constexpr (PAGED) {
        pg_v = lds_s32_now(sbase + C::kOffTab + 4u * (i % kPageSlots));
        pg_k = lds_s32_now(sbase + C::kOffTab + 4u * ((i + kKStages) % kPageSlots));
      }
      const float* wb = wmax + (i & 1) * kWarps * G;
      float mt = lane < n_dec ? wb[lane] : NEG_INF;
      if constexpr (G == 8) mt = fmaxf(mt, wb[lane + 32]);
#pragma unroll
      for (int o = G; o < n_dec; o <<= 1) mt = fmaxf(mt, __shfl_xor_sync(FULL, mt, o));
      // row lane % G passes iff it has a history and the tile max is below m - tau
      const bool pass =
          lane >= n_dec || (m_exact != NEG_INF && (mt == NEG_INF || mt < m_exact - tau_log2));
      keep_i = !SKIP || !__all_sync(FULL, pass);
      // per-head rule: bit r set iff row r computes this tile (lanes 0..G-1 hold rows 0..G-1)
      unsigned row_keep = 0xffffffffu;
      if constexpr (per_head && SKIP) row_keep = __ballot_sync(FULL, !pass);
      m_exact = fmaxf(m_exact, mt);  // a skipped tile never raises it
      if (keep_i) {
        const bool moved = m_exact > m_ref + kRefSlack;
        if (__any_sync(FULL, moved)) {
          const float ref_new = moved ? m_exact : m_ref;
          const float sc = moved ? ex2(m_ref - ref_new) : 1.f;  // m_ref = -inf gives 0
          lsum *= __shfl_sync(FULL, sc, row_q);
          m_ref = ref_new;
          if (warp == 0 && lane < G) ref_ring[(i % kPRing) * 8 + lane] = ref_new;
          if (tid == 0) flag_ring[i % kPRing] = 1;
        } else if (tid == 0) {
          flag_ring[i % kPRing] = 0;
        }
        // probabilities of tile i relative to the reference max of each row
        const float mr = __shfl_sync(FULL, m_ref, row_q);
        float* pr = p_ring + (i % kPRing) * kDecodeTile * G;
#pragma unroll
        for (int it = 0; it < C::kSIters; ++it) {
          const int key = warp * C::kKeysPerWarp + it * C::kKPI + kl;
          float p = ex2(sv[it] - mr);
          if constexpr (per_head) p = ((row_keep >> row_q) & 1u) ? p : 0.f;
          if (leader) {
            pr[key * G + row_q] = p;
            lsum += p;
          }
        }
      }
      if (per_head && skip_mask && warp == 0 && lane < G)  // one mask entry per query head
        skip_mask[(static_cast<size_t>(b) * Hq + kv * G + lane) * n_tiles_all + t_begin + i] =
            (keep_i && ((row_keep >> lane) & 1u)) ? 0 : 1;
      if (tid == 0) {
        const int t = t_begin + i;
        if (skip_mask && !per_head) skip_mask[static_cast<size_t>(bh) * n_tiles_all + t] = keep_i ? 0 : 1;
        if (keep_i) {  // the slot's previous tile finished its P*V before this barrier
          const int vs = v_issued % kVStages;
          // test support: the first copy can be withheld, so that every wait
          // for it runs out and the timeout path is exercised
          if (!(withhold_v && v_issued == 0))
            issue(sbase + C::kOffV + vs * C::kTileBytes, &tmV, b_v_full(vs), t, pg_v);
          ++v_issued;
        }
        if (i + kKStages < nt) {  // every thread has finished reading K slot i % kKStages
          const int ks = i % kKStages;
          issue(sbase + C::kOffK + ks * C::kTileBytes, &tmK, b_k_full(ks), t + kKStages, pg_k);
          ++k_issued;
        }
      }
      // chunk c = i / kPageChunk starts: stage chunk c + 1 into the slots of
      // chunk c - 1, whose last copy (tile i - 1's V) was issued before the
      // barrier above; chunk c + 1 is first read kPageChunk - kKStages
      // barriers later
      if (PAGED && i >= kPageChunk && i % kPageChunk == 0) stage_pages(i + kPageChunk);
    }
    kept_bits = (kept_bits << 1) | (keep_i ? 1u : 0u);

    // ---------------- C: P*V of tile t = i - kLag (its p were written kLag barriers ago)
    const int t = i - kLag;
    if (t >= 0 && ((kept_bits >> kLag) & 1u)) {
      const int vs = pv_count % kVStages;
      const bool got = mbar_wait(b_v_full(vs), (pv_count / kVStages) & 1, never, wait_limit_ns);
      ok = ok && got;  // acted on at the next barrier
      if (got) {
        if (flag_ring[t % kPRing]) {  // move the sums to this tile's reference max
          float rn[G];
          load_row_floats<G>(ref_ring + (t % kPRing) * 8, rn);
#pragma unroll
          for (int r = 0; r < G; ++r) {
            if (rn[r] != m_acc[r]) {
              const float a = ex2(m_acc[r] - rn[r]);  // m_acc = -inf initially gives 0
              const float2 a2 = make_float2(a, a);
#pragma unroll
              for (int e = 0; e < 4; ++e) acc[r][e] = __fmul2_rn(acc[r][e], a2);
              m_acc[r] = rn[r];
            }
          }
        }
        const uint8_t* vt = smem + C::kOffV + vs * C::kTileBytes;
        const float* pr = p_ring + (t % kPRing) * kDecodeTile * G;
        // contiguous cache: rows past L arrive as zeros (with p = 0); paged:
        // rows past the end of the sequence are whatever the page holds (even
        // NaN), so in a sequence's last, partial tile those keys (p = 0) read
        // the last valid row instead.  Full tiles take the loop with
        // compile-time key offsets.
        auto pv_keys = [&](auto clamp) {
          const int key_last_v = Lb - (t_begin + t) * kDecodeTile - 1;
#pragma unroll
          for (int e2 = 0; e2 < C::kVKeys; ++e2) {
            const int key = kg + C::kGroups * e2;
            const int key_ld = decltype(clamp)::value ? min(key, key_last_v) : key;
            const uint4 u = *reinterpret_cast<const uint4*>(vt + chunk_off<D>(key_ld, ch));
            float2 vf[4];
            bf16x8_to_f32(u, vf);
            float pv[G];
            load_row_floats<G>(pr + key * G, pv);
#pragma unroll
            for (int r = 0; r < G; ++r) {
              const float2 p2 = make_float2(pv[r], pv[r]);
#pragma unroll
              for (int e = 0; e < 4; ++e) acc[r][e] = __ffma2_rn(p2, vf[e], acc[r][e]);
            }
          }
        };
        if (PAGED && Lb - (t_begin + t) * kDecodeTile < kDecodeTile)
          pv_keys(std::integral_constant<bool, true>{});
        else
          pv_keys(std::integral_constant<bool, false>{});
      }
      ++pv_count;
    }
  }

  // a V wait in the last iterations may have failed after the last barrier
  if (__syncthreads_or(!ok)) {
    // leave no bulk copy in flight into this CTA's shared memory: the last
    // copy issued into each ring slot is waited for (earlier ones in the same
    // slot completed before it was reused)
    if (tid == 0) {
      atomicCAS(status, 0, ATTN_DEVICE_TIMEOUT_BASE + 20);
      for (int k = max(0, k_issued - kKStages); k < k_issued; ++k)
        mbar_drain(b_k_full(k % kKStages), (k / kKStages) & 1, wait_limit_ns);
      for (int k = max(0, v_issued - kVStages); k < v_issued; ++k)
        if (!(withhold_v && k == 0))  // a withheld copy was never issued
          mbar_drain(b_v_full(k % kVStages), (k / kVStages) & 1, wait_limit_ns);
      if (seed_issued) mbar_drain(b_seed, 0, wait_limit_ns);
    }
    // this split's partials are written as an empty split (zero weight in the
    // merge), so the output never mixes in scratch left by an earlier call
    for (int idx = tid; idx < G * D; idx += kDecThreads) {
      const size_t row = static_cast<size_t>(b) * Hq + kv * G + idx / D;
      o_part[(row * n_splits + split) * D + idx % D] = 0.f;
    }
    if (tid < G) lse_part[(static_cast<size_t>(b) * Hq + kv * G + tid) * n_splits + split] = NEG_INF;
    return;
  }

  // ---------------- combine the key subsets: lanes of one warp, then warps
#pragma unroll
  for (int o = C::kChunks; o < 32; o <<= 1) {
#pragma unroll
    for (int r = 0; r < G; ++r) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[r][e].x += __shfl_xor_sync(FULL, acc[r][e].x, o);
        acc[r][e].y += __shfl_xor_sync(FULL, acc[r][e].y, o);
      }
    }
  }
  float lrow[G];  // sum of p over the warp's keys, per row
#pragma unroll
  for (int r = 0; r < G; ++r) {
    float x = row_q == r ? lsum : 0.f;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) x += __shfl_xor_sync(FULL, x, o);
    lrow[r] = x;
  }
  // every copy has landed and been read: the K ring is free for the reduction
  float* red = reinterpret_cast<float*>(smem + C::kOffK);  // [warp][G][D]
  if (lane < C::kChunks) {
#pragma unroll
    for (int r = 0; r < G; ++r) {
      float4* dst = reinterpret_cast<float4*>(red + (warp * G + r) * D + ch * 8);
      dst[0] = make_float4(acc[r][0].x, acc[r][0].y, acc[r][1].x, acc[r][1].y);
      dst[1] = make_float4(acc[r][2].x, acc[r][2].y, acc[r][3].x, acc[r][3].y);
    }
  }
  if (lane == 0) {
#pragma unroll
    for (int r = 0; r < G; ++r) wl[warp * G + r] = lrow[r];
  }
  __syncthreads();
  for (int idx = tid; idx < G * D; idx += kDecThreads) {
    const int r = idx / D, col = idx % D;
    float s = 0.f, den = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      s += red[(w * G + r) * D + col];
      den += wl[w * G + r];
    }
    const size_t row = static_cast<size_t>(b) * Hq + kv * G + r;
    // a row that skipped every tile of its split (possible with the sink seed
    // or the per-head rule) contributes nothing to the merge
    o_part[(row * n_splits + split) * D + col] = den > 0.f ? s / den : 0.f;
  }
  if (tid < G) {
    // lane tid of warp 0 holds the reference max of row tid, which is the one
    // both the sums of p and the P*V sums are relative to
    float den = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) den += wl[w * G + tid];
    const size_t row = static_cast<size_t>(b) * Hq + kv * G + tid;
    lse_part[row * n_splits + split] = den > 0.f ? m_ref + __log2f(den) : NEG_INF;
  }
}

// Exact merge of the split partials: o = sum_s 2^{lse_s - M} o_s / sum_s 2^{lse_s - M}.
template <int D>
__global__ void __launch_bounds__(D)
    decode_combine_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part,
                          __nv_bfloat16* __restrict__ o, int n_splits) {
  const int row = blockIdx.x;
  const int col = threadIdx.x;
  const float* lse = lse_part + static_cast<size_t>(row) * n_splits;
  float M = -__int_as_float(0x7f800000);
  for (int s = 0; s < n_splits; ++s) M = fmaxf(M, lse[s]);
  float num = 0.f, den = 0.f;
  for (int s = 0; s < n_splits; ++s) {
    const float w = ex2(lse[s] - M);
    den += w;
    num = fmaf(w, o_part[(static_cast<size_t>(row) * n_splits + s) * D + col], num);
  }
  // every split empty (only after a wait gave up): 0 rather than NaN
  o[static_cast<size_t>(row) * D + col] = __float2bfloat16_rn(den > 0.f ? num / den : 0.f);
}

namespace {

PFN_cuTensorMapEncodeTiled_v12000 dec_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult qr;
    void* p = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// [B*Hkv, L, D] bf16, d fastest; box = 64 columns x 64 keys, 128-byte swizzle,
// out-of-range keys read as zeros
bool dec_map(CUtensorMap* m, const void* base, int BH, int L, int D) {
  auto enc = dec_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(L),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(L) * D * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(kDecodeTile), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int G, int RULE, bool PAGED, bool SKIP>
int launch_dgrp(const DecodeLaunch& a) {
  using C = DecCfg<D, G>;
  auto kern = decode_partial_kernel<D, G, RULE, PAGED, SKIP>;
  constexpr int smem_bytes = PAGED ? C::kSmemBytesPaged : C::kSmemBytes;
  static uint64_t attr_done = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  if (dev < 64 && !(attr_done >> dev & 1)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes) !=
        cudaSuccess)
      return ATTN_ERR_CUDA;
    attr_done |= uint64_t(1) << dev;
  }
  CUtensorMap mk, mv;
  if (PAGED) {  // the page pool as [num_pages * Hkv, 64, D]
    if (!dec_map(&mk, a.K, a.num_pages * a.Hkv, kDecodeTile, D) ||
        !dec_map(&mv, a.V, a.num_pages * a.Hkv, kDecodeTile, D))
      return ATTN_ERR_CUDA;
  } else if (!dec_map(&mk, a.K, a.B * a.Hkv, a.L, D) || !dec_map(&mv, a.V, a.B * a.Hkv, a.L, D)) {
    return ATTN_ERR_CUDA;
  }
  dim3 grid(a.n_splits, a.Hkv, a.B);
  kern<<<grid, kDecThreads, smem_bytes, a.stream>>>(
      mk, mv, static_cast<const __nv_bfloat16*>(a.q), a.o_part, a.lse_part, a.skip_mask,
      a.status, a.Hq, a.Hkv, a.L, a.split_len, a.n_splits, a.scale_log2, a.tau_log2,
      a.wait_limit_ns, a.withhold_v, a.block_table, a.seq_lens, a.max_pages);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  decode_combine_kernel<D><<<a.B * a.Hq, D, 0, a.stream>>>(
      a.o_part, a.lse_part, static_cast<__nv_bfloat16*>(a.o), a.n_splits);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <int D, int G, int RULE>
int launch_dgr(const DecodeLaunch& a) {
  if (a.tau_is_inf)
    return a.block_table ? launch_dgrp<D, G, RULE, true, false>(a) : launch_dgrp<D, G, RULE, false, false>(a);
  return a.block_table ? launch_dgrp<D, G, RULE, true, true>(a) : launch_dgrp<D, G, RULE, false, true>(a);
}

template <int D, int G>
int launch_dg(const DecodeLaunch& a) {
  switch (a.rule) {
    case 0: return launch_dgr<D, G, 0>(a);
    case ATTN_DECODE_RULE_PER_HEAD: return launch_dgr<D, G, ATTN_DECODE_RULE_PER_HEAD>(a);
    case ATTN_DECODE_RULE_SINK_SEED: return launch_dgr<D, G, ATTN_DECODE_RULE_SINK_SEED>(a);
    case ATTN_DECODE_RULE_PER_HEAD | ATTN_DECODE_RULE_SINK_SEED:
      return launch_dgr<D, G, ATTN_DECODE_RULE_PER_HEAD | ATTN_DECODE_RULE_SINK_SEED>(a);
    default: return ATTN_ERR_INVALID_ARG;
  }
}

template <int D>
int launch_d(const DecodeLaunch& a) {
  switch (a.Hq / a.Hkv) {
    case 1: return launch_dg<D, 1>(a);
    case 2: return launch_dg<D, 2>(a);
    case 4: return launch_dg<D, 4>(a);
    case 8: return launch_dg<D, 8>(a);
    default: return ATTN_ERR_UNSUPPORTED;
  }
}

}  // namespace

int launch_decode(const DecodeLaunch& a) {
  if (a.d == 64) return launch_d<64>(a);
  if (a.d == 128) return launch_d<128>(a);
  return ATTN_ERR_INVALID_ARG;
}

}  // namespace bss
