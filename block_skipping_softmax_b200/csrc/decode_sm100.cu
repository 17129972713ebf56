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
// Decode is bound by HBM reads of K and V, so the kernel is built around the
// memory system rather than the tensor cores (a g-row GEMV does not fill an
// MMA): every K tile is one contiguous 16 KB (d=128) bulk copy into a shared-
// memory ring, issued three tiles ahead; a V tile is requested only once the
// tile is known to be kept, and consumed two iterations later so its latency
// stays hidden.  Shared memory is read with 16-byte vector loads, each warp
// instruction covering whole key rows; dot products use packed fp32 FMAs and
// a transposing butterfly reduction across the lanes of one key.
//
// One CTA barrier per tile: the scores of tile i and each warp's per-row
// maxima are formed before it; after it every thread takes the same skip
// decision from the eight warp maxima (no serial phase), the lanes that hold
// scores turn them into probabilities for a later P*V, and thread 0 refills
// the copy rings.  Output per split: normalised partial o (fp32) and its
// log2-sum-exp; a second kernel merges the splits exactly.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

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

template <int D, int G>
struct DecCfg {
  static constexpr int kTileBytes = kDecodeTile * D * 2;
  static constexpr int kCPK = D / 8;                  // 16-byte chunks per key row
  static constexpr int kKPI = 32 / kCPK;              // keys per warp instruction
  static constexpr int kKeysPerWarp = kDecodeTile / kWarps;
  static constexpr int kIters = kKeysPerWarp / kKPI;
  static constexpr int kLanesPerRow = kCPK / G;       // lanes holding copies of one score
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kKStages * kTileBytes;
  static constexpr int kOffP = kOffV + kVStages * kTileBytes;             // float [PR][64][G]
  static constexpr int kOffW = kOffP + kPRing * kDecodeTile * G * 4;      // float [2][warps][G]
  static constexpr int kOffMisc = kOffW + 2 * kWarps * G * 4;
  static constexpr int kOffBar = kOffMisc + 64;                           // k_full, v_full
  static constexpr int kSmemBytes = kOffBar + 8 * (kKStages + kVStages) + 128;
  // the final cross-warp reduction reuses the K ring
  static_assert(kWarps * G * (D + 1) * 4 <= kKStages * kTileBytes, "reduction scratch");
  static_assert(G <= kCPK, "rows per group");
};

}  // namespace

template <int D, int G>
__global__ void __launch_bounds__(kDecThreads, (G <= 4) ? 2 : 1)
    decode_partial_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ K,
                          const __nv_bfloat16* __restrict__ V, float* __restrict__ o_part,
                          float* __restrict__ lse_part, uint8_t* __restrict__ skip_mask,
                          int* __restrict__ status, int Hq, int Hkv, int L, int split_len,
                          int n_splits, float scale_log2, float tau_log2, int tau_is_inf,
                          unsigned long long wait_limit_ns) {
  using C = DecCfg<D, G>;
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  float* p_ring = reinterpret_cast<float*>(smem + C::kOffP);
  float* wmax = reinterpret_cast<float*>(smem + C::kOffW);
  // Give-ups are made CTA-uniform with __syncthreads_or, so no role ever
  // needs to be told to stop early: this flag stays 0.
  volatile int* never = reinterpret_cast<volatile int*>(smem + C::kOffMisc);
  const uint32_t bar0 = sbase + C::kOffBar;
  auto b_k_full = [&](int s) { return bar0 + 8u * s; };
  auto b_v_full = [&](int s) { return bar0 + 8u * (kKStages + s); };

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int split = blockIdx.x;
  const int kv = blockIdx.y;
  const int b = blockIdx.z;
  const int n_tiles_all = (L + kDecodeTile - 1) / kDecodeTile;
  const int t_begin = split * (split_len / kDecodeTile);
  const int t_end = min(n_tiles_all, t_begin + split_len / kDecodeTile);
  const int nt = t_end - t_begin;
  const size_t kv_off = (static_cast<size_t>(b) * Hkv + kv) * static_cast<size_t>(L) * D;
  const __nv_bfloat16* Kg = K + kv_off;
  const __nv_bfloat16* Vg = V + kv_off;
  const float NEG_INF = -__int_as_float(0x7f800000);

  auto tile_bytes = [&](int t) {  // the last tile of the sequence may be ragged
    const int keys = min(kDecodeTile, L - t * kDecodeTile);
    return static_cast<uint32_t>(keys * D * 2);
  };

  if (tid == 0) {
    for (int s = 0; s < kKStages; ++s) mbar_init(b_k_full(s), 1);
    for (int s = 0; s < kVStages; ++s) mbar_init(b_v_full(s), 1);
    *never = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  __syncthreads();
  int k_issued = 0, v_issued = 0;
  if (tid == 0) {
    for (int i = 0; i < kKStages && i < nt; ++i) {
      const int t = t_begin + i;
      mbar_arrive_expect_tx(b_k_full(i), tile_bytes(t));
      bulk_load(sbase + C::kOffK + i * C::kTileBytes, Kg + static_cast<size_t>(t) * kDecodeTile * D,
                tile_bytes(t), b_k_full(i));
      ++k_issued;
    }
  }

  // this lane's slice: 16-byte chunk `c` of key `sub` within each warp instruction
  const int c = lane % C::kCPK;
  const int sub = lane / C::kCPK;
  const int my_row = c / C::kLanesPerRow;  // the score row this lane ends up holding
  const bool writer = (c % C::kLanesPerRow) == 0;
  float2 qf[G][4];
#pragma unroll
  for (int r = 0; r < G; ++r) {
    const uint4 u = *reinterpret_cast<const uint4*>(
        q + (static_cast<size_t>(b) * Hq + kv * G + r) * D + c * 8);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e)
      qf[r][e] = make_float2(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xffff0000u));
  }
  float2 acc[G][4];
  float lsum[G];
  // every thread keeps identical copies of the decision state
  float m_exact[G];           // exact running max after the latest tested tile (log2 units)
  float m_hist[kLag + 1][G];  // m_hist[k][r] = running max after tile i - k
  float m_acc[G];             // reference max of the partial sums acc / lsum
#pragma unroll
  for (int r = 0; r < G; ++r) {
    lsum[r] = 0.f;
    m_exact[r] = NEG_INF;
    m_acc[r] = NEG_INF;
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[r][e] = make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k <= kLag; ++k) m_hist[k][r] = NEG_INF;
  }
  uint32_t kept_bits = 0;  // bit k: tile i - k was kept
  int pv_count = 0;        // V tiles consumed
  bool ok = true;          // this thread's waits so far succeeded

  for (int i = 0; i < nt + kLag; ++i) {
    // ---------------- A: scores of tile i and the per-warp row maxima
    float sv[C::kIters];
    if (i < nt) {
      const int ks = i % kKStages;
      const bool got = mbar_wait(b_k_full(ks), (i / kKStages) & 1, never, wait_limit_ns);
      ok = ok && got;
      const uint8_t* kt = smem + C::kOffK + ks * C::kTileBytes;
      const int key_lim = L - (t_begin + i) * kDecodeTile;  // keys >= key_lim are past L
      float wm = NEG_INF;
#pragma unroll
      for (int it = 0; it < C::kIters; ++it) {
        const int key = warp * C::kKeysPerWarp + it * C::kKPI + sub;
        float v[G];
        if (got) {
          const uint4 u = *reinterpret_cast<const uint4*>(kt + key * D * 2 + c * 16);
          const uint32_t w[4] = {u.x, u.y, u.z, u.w};
          float2 kf[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            kf[e] = make_float2(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xffff0000u));
#pragma unroll
          for (int r = 0; r < G; ++r) {
            float2 s2 = __fmul2_rn(qf[r][0], kf[0]);
#pragma unroll
            for (int e = 1; e < 4; ++e) s2 = __ffma2_rn(qf[r][e], kf[e], s2);
            v[r] = s2.x + s2.y;
          }
        } else {
#pragma unroll
          for (int r = 0; r < G; ++r) v[r] = 0.f;
        }
        // transposing butterfly over the kCPK lanes of this key: each halving
        // step keeps half of the rows, so after log2(G) steps a lane owns one
        // row (my_row); the remaining steps are plain sums
#pragma unroll
        for (int step = 0; (C::kCPK >> (step + 1)) >= 1; ++step) {
          const int o = C::kCPK >> (step + 1);
          const int n = G >> step;
          if (n > 1) {
            const int hh = n / 2;
            const bool upper = (lane & o) != 0;
#pragma unroll
            for (int r = 0; r < hh; ++r) {
              const float send = upper ? v[r] : v[r + hh];
              const float keep = upper ? v[r + hh] : v[r];
              v[r] = keep + __shfl_xor_sync(0xffffffffu, send, o);
            }
          } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
          }
        }
        sv[it] = key < key_lim ? v[0] * scale_log2 : NEG_INF;
        wm = fmaxf(wm, sv[it]);
      }
      // max over this warp's keys for my_row: combine the `sub` lanes
#pragma unroll
      for (int o = C::kCPK; o < 32; o <<= 1) wm = fmaxf(wm, __shfl_xor_sync(0xffffffffu, wm, o));
      if (writer && sub == 0) wmax[((i & 1) * kWarps + warp) * G + my_row] = wm;
    }
    if (__syncthreads_or(!ok)) {  // the single per-tile barrier; also a uniform give-up
      ok = false;
      break;
    }
    // ---------------- B: decision for tile i (the same in every thread)
    bool keep_i = false;
    if (i < nt) {
      bool all_pass = !tau_is_inf;
#pragma unroll
      for (int r = 0; r < G; ++r) {
        float mt = NEG_INF;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) mt = fmaxf(mt, wmax[((i & 1) * kWarps + w) * G + r]);
        const bool pass = m_exact[r] != NEG_INF && (mt == NEG_INF || mt < m_exact[r] - tau_log2);
        all_pass = all_pass && pass;
        m_exact[r] = fmaxf(m_exact[r], mt);
      }
      keep_i = !all_pass;
      if (tid == 0) {
        const int t = t_begin + i;
        if (skip_mask)
          skip_mask[(static_cast<size_t>(b) * Hkv + kv) * n_tiles_all + t] = keep_i ? 0 : 1;
        if (keep_i) {  // the slot's previous tile finished its P*V before this barrier
          const int vs = v_issued % kVStages;
          mbar_arrive_expect_tx(b_v_full(vs), tile_bytes(t));
          bulk_load(sbase + C::kOffV + vs * C::kTileBytes,
                    Vg + static_cast<size_t>(t) * kDecodeTile * D, tile_bytes(t), b_v_full(vs));
          ++v_issued;
        }
        if (i + kKStages < nt) {  // every thread has finished reading K slot i % kKStages
          const int ks = i % kKStages;
          const int tn = t + kKStages;
          mbar_arrive_expect_tx(b_k_full(ks), tile_bytes(tn));
          bulk_load(sbase + C::kOffK + ks * C::kTileBytes,
                    Kg + static_cast<size_t>(tn) * kDecodeTile * D, tile_bytes(tn), b_k_full(ks));
          ++k_issued;
        }
      }
      // probabilities of tile i relative to the running max after tile i
      if (keep_i && writer) {
        float* pr = p_ring + (i % kPRing) * kDecodeTile * G;
        float mr = NEG_INF;
#pragma unroll
        for (int r = 0; r < G; ++r)
          if (r == my_row) mr = m_exact[r];
#pragma unroll
        for (int it = 0; it < C::kIters; ++it) {
          const int key = warp * C::kKeysPerWarp + it * C::kKPI + sub;
          pr[key * G + my_row] = ex2(sv[it] - mr);
        }
      }
    }
    // shift the per-tile history: running max after tile i, kept bit of tile i
#pragma unroll
    for (int k = kLag; k >= 1; --k)
#pragma unroll
      for (int r = 0; r < G; ++r) m_hist[k][r] = m_hist[k - 1][r];
#pragma unroll
    for (int r = 0; r < G; ++r) m_hist[0][r] = m_exact[r];
    kept_bits = (kept_bits << 1) | (keep_i ? 1u : 0u);

    // ---------------- C: P*V of tile t = i - kLag (its p were written kLag barriers ago)
    const int t = i - kLag;
    if (t >= 0 && ((kept_bits >> kLag) & 1u)) {
      const int vs = pv_count % kVStages;
      const bool got = mbar_wait(b_v_full(vs), (pv_count / kVStages) & 1, never, wait_limit_ns);
      ok = ok && got;  // acted on at the next barrier
      if (got) {
        // move the reference max of the partial sums up to this tile's
#pragma unroll
        for (int r = 0; r < G; ++r) {
          const float mn = m_hist[kLag][r];
          if (mn != m_acc[r]) {
            const float a = ex2(m_acc[r] - mn);  // m_acc = -inf initially gives 0
            lsum[r] *= a;
            const float2 a2 = make_float2(a, a);
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[r][e] = __fmul2_rn(acc[r][e], a2);
            m_acc[r] = mn;
          }
        }
        const uint8_t* vt = smem + C::kOffV + vs * C::kTileBytes;
        const float* pr = p_ring + (t % kPRing) * kDecodeTile * G;
        const int key_lim = L - (t_begin + t) * kDecodeTile;
#pragma unroll
        for (int it = 0; it < C::kIters; ++it) {
          const int key = warp * C::kKeysPerWarp + it * C::kKPI + sub;
          if (key < key_lim) {
            const uint4 u = *reinterpret_cast<const uint4*>(vt + key * D * 2 + c * 16);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
            float2 vf[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              vf[e] = make_float2(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xffff0000u));
#pragma unroll
            for (int r = 0; r < G; ++r) {
              const float pv = pr[key * G + r];
              const float2 p2 = make_float2(pv, pv);
#pragma unroll
              for (int e = 0; e < 4; ++e) acc[r][e] = __ffma2_rn(p2, vf[e], acc[r][e]);
              if (c == 0) lsum[r] += pv;
            }
          }
        }
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
        mbar_drain(b_v_full(k % kVStages), (k / kVStages) & 1, wait_limit_ns);
    }
    return;
  }

  // ---------------- reduce the partial sums: lanes of one chunk, then warps
#pragma unroll
  for (int o = C::kCPK; o < 32; o <<= 1) {
#pragma unroll
    for (int r = 0; r < G; ++r) {
      lsum[r] += __shfl_xor_sync(0xffffffffu, lsum[r], o);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[r][e].x += __shfl_xor_sync(0xffffffffu, acc[r][e].x, o);
        acc[r][e].y += __shfl_xor_sync(0xffffffffu, acc[r][e].y, o);
      }
    }
  }
  float* red = reinterpret_cast<float*>(smem + C::kOffK);  // [warp][G][D+1]
  __syncthreads();
  if (sub == 0) {
#pragma unroll
    for (int r = 0; r < G; ++r) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        red[(warp * G + r) * (D + 1) + c * 8 + 2 * e] = acc[r][e].x;
        red[(warp * G + r) * (D + 1) + c * 8 + 2 * e + 1] = acc[r][e].y;
      }
      if (c == 0) red[(warp * G + r) * (D + 1) + D] = lsum[r];
    }
  }
  __syncthreads();
  for (int idx = tid; idx < G * (D + 1); idx += kDecThreads) {
    const int r = idx / (D + 1), col = idx % (D + 1);
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) s += red[(w * G + r) * (D + 1) + col];
    red[r * (D + 1) + col] = s;  // warp 0's slot; only this thread touches (r, col)
  }
  __syncthreads();
  for (int idx = tid; idx < G * D; idx += kDecThreads) {
    const int r = idx / D, col = idx % D;
    const size_t row = static_cast<size_t>(b) * Hq + kv * G + r;
    o_part[(row * n_splits + split) * D + col] = red[r * (D + 1) + col] / red[r * (D + 1) + D];
  }
  if (tid < G) {
    // every thread holds the same reference max (skipped tiles never move the
    // running max, so it is the value used by the last P*V); select it with a
    // constant index
    float mr = NEG_INF;
#pragma unroll
    for (int r = 0; r < G; ++r)
      if (r == tid) mr = m_acc[r];
    const size_t row = static_cast<size_t>(b) * Hq + kv * G + tid;
    lse_part[row * n_splits + split] = mr + __log2f(red[tid * (D + 1) + D]);
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
  o[static_cast<size_t>(row) * D + col] = __float2bfloat16_rn(num / den);
}

namespace {

template <int D, int G>
int launch_dg(const DecodeLaunch& a) {
  using C = DecCfg<D, G>;
  auto kern = decode_partial_kernel<D, G>;
  static uint64_t attr_done = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  if (dev < 64 && !(attr_done >> dev & 1)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
        cudaSuccess)
      return ATTN_ERR_CUDA;
    attr_done |= uint64_t(1) << dev;
  }
  dim3 grid(a.n_splits, a.Hkv, a.B);
  kern<<<grid, kDecThreads, C::kSmemBytes, a.stream>>>(
      static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.K),
      static_cast<const __nv_bfloat16*>(a.V), a.o_part, a.lse_part, a.skip_mask, a.status, a.Hq,
      a.Hkv, a.L, a.split_len, a.n_splits, a.scale_log2, a.tau_log2, a.tau_is_inf,
      a.wait_limit_ns);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  decode_combine_kernel<D><<<a.B * a.Hq, D, 0, a.stream>>>(
      a.o_part, a.lse_part, static_cast<__nv_bfloat16*>(a.o), a.n_splits);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
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
