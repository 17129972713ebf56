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
// instruction covering whole key rows (conflict-free); dot products use fp32
// FMAs and a transposing butterfly reduction across the lanes of one key.
// Output per split: normalised partial o (fp32) and its log2-sum-exp; a
// second kernel merges the splits exactly.
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
constexpr int kKStages = 3;   // K tiles in flight ahead of the compute
constexpr int kLag = 2;       // a kept tile's P*V runs kLag iterations after its test
constexpr int kVStages = kLag + 1;
constexpr int kSRing = kLag + 1;
constexpr int kDRing = 4;

template <int D, int G>
struct DecCfg {
  static constexpr int kTileBytes = kDecodeTile * D * 2;
  static constexpr int kCPK = D / 8;          // 16-byte chunks per key row
  static constexpr int kKPI = 32 / kCPK;      // keys per warp instruction
  static constexpr int kIters = (kDecodeTile / kWarps) / kKPI;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kKStages * kTileBytes;
  static constexpr int kOffS = kOffV + kVStages * kTileBytes;             // float [SR][G][64]
  static constexpr int kOffP = kOffS + kSRing * G * kDecodeTile * 4;      // float [64][G]
  static constexpr int kOffM = kOffP + kDecodeTile * G * 4;               // float [G]
  static constexpr int kOffDec = kOffM + 64;                              // int [kDRing]
  static constexpr int kOffBar = kOffDec + 64;                            // k_full, v_full
  static constexpr int kSmemBytes = kOffBar + 8 * (kKStages + kVStages) + 128;
  // the final cross-warp reduction reuses the K ring
  static_assert(kWarps * G * (D + 1) * 4 <= kKStages * kTileBytes, "reduction scratch");
};

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

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
  float* s_ring = reinterpret_cast<float*>(smem + C::kOffS);
  float* p_sm = reinterpret_cast<float*>(smem + C::kOffP);
  float* m_sm = reinterpret_cast<float*>(smem + C::kOffM);
  volatile int* dec = reinterpret_cast<volatile int*>(smem + C::kOffDec);
  // Give-ups in this kernel are made CTA-uniform with __syncthreads_or, so no
  // role ever needs to be told to stop early: the flag stays 0.
  volatile int* never = reinterpret_cast<volatile int*>(smem + C::kOffDec + 32);
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
  float qf[G][8];
#pragma unroll
  for (int r = 0; r < G; ++r) {
    const uint4 u = *reinterpret_cast<const uint4*>(
        q + (static_cast<size_t>(b) * Hq + kv * G + r) * D + c * 8);
    bf16x8_to_f32(u, qf[r]);
  }
  float acc[G][8];
  float lsum[G];
  float m_used[G];
#pragma unroll
  for (int r = 0; r < G; ++r) {
    lsum[r] = 0.f;
    m_used[r] = NEG_INF;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[r][e] = 0.f;
  }
  float m_exact[G];  // exact running max of each row (warp 0 keeps it)
#pragma unroll
  for (int r = 0; r < G; ++r) m_exact[r] = NEG_INF;
  int kept_issue = 0;  // V tiles requested (thread 0)
  int pv_count = 0;    // V tiles consumed
  bool ok = true;
  int k_consumed = 0;

  for (int i = 0; i < nt + kLag; ++i) {
    // ---------------- scores of tile i: s = q . k (log2 units) into the ring
    if (i < nt) {
      const int ks = i % kKStages;
      ok = mbar_wait(b_k_full(ks), (i / kKStages) & 1, never, wait_limit_ns);
    }
    if (__syncthreads_or(!ok)) {  // uniform give-up
      ok = false;
      break;
    }
    if (i < nt) {
      const int ks = i % kKStages;
      const uint8_t* kt = smem + C::kOffK + ks * C::kTileBytes;
      float* srow = s_ring + (i % kSRing) * G * kDecodeTile;
      const int key_lim = L - (t_begin + i) * kDecodeTile;  // keys >= key_lim are past L
#pragma unroll
      for (int it = 0; it < C::kIters; ++it) {
        const int key = warp * (kDecodeTile / kWarps) + it * C::kKPI + sub;
        const uint4 u = *reinterpret_cast<const uint4*>(kt + key * D * 2 + c * 16);
        float kf[8];
        bf16x8_to_f32(u, kf);
        float v[G];
#pragma unroll
        for (int r = 0; r < G; ++r) {
          float sacc = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) sacc = fmaf(qf[r][e], kf[e], sacc);
          v[r] = sacc;
        }
        // transposing butterfly over the kCPK lanes of this key: each halving
        // step keeps half of the rows, so after log2(G) steps a lane owns one
        // row (row = c / (kCPK/G)); the remaining steps are plain sums
#pragma unroll
        for (int step = 0; (C::kCPK >> (step + 1)) >= 1; ++step) {
          const int o = C::kCPK >> (step + 1);  // xor distance of this step
          const int n = G >> step;               // rows this lane still holds (if >= 1)
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
        constexpr int kLanesPerRow = C::kCPK / G;
        if ((c % kLanesPerRow) == 0) {
          const int r = c / kLanesPerRow;
          srow[r * kDecodeTile + key] = key < key_lim ? v[0] * scale_log2 : NEG_INF;
        }
      }
      ++k_consumed;
    }
    __syncthreads();  // S1: scores visible, K slot free
    // ---------------- skip test for tile i (warp 0), then refill the rings
    if (warp == 0 && i < nt) {
      const float* srow = s_ring + (i % kSRing) * G * kDecodeTile;
      bool all_pass = !tau_is_inf;
#pragma unroll
      for (int r = 0; r < G; ++r) {
        float mt = fmaxf(srow[r * kDecodeTile + lane], srow[r * kDecodeTile + lane + 32]);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o));
        const bool pass = m_exact[r] != NEG_INF && (mt == NEG_INF || mt < m_exact[r] - tau_log2);
        all_pass = all_pass && pass;
        m_exact[r] = fmaxf(m_exact[r], mt);
      }
      const bool skip = all_pass;
      if (lane == 0) {
#pragma unroll
        for (int r = 0; r < G; ++r) m_sm[r] = m_exact[r];
        dec[i % kDRing] = skip ? 0 : 1;
        if (skip_mask)
          skip_mask[(static_cast<size_t>(b) * Hkv + kv) * n_tiles_all + t_begin + i] = skip ? 1 : 0;
        const int t = t_begin + i;
        if (!skip) {
          const int vs = kept_issue % kVStages;
          mbar_arrive_expect_tx(b_v_full(vs), tile_bytes(t));
          bulk_load(sbase + C::kOffV + vs * C::kTileBytes,
                    Vg + static_cast<size_t>(t) * kDecodeTile * D, tile_bytes(t), b_v_full(vs));
          ++kept_issue;
          ++v_issued;
        }
        if (i + kKStages < nt) {
          const int ks = i % kKStages;
          const int tn = t + kKStages;
          mbar_arrive_expect_tx(b_k_full(ks), tile_bytes(tn));
          bulk_load(sbase + C::kOffK + ks * C::kTileBytes,
                    Kg + static_cast<size_t>(tn) * kDecodeTile * D, tile_bytes(tn), b_k_full(ks));
          ++k_issued;
        }
      }
    }
    __syncthreads();  // S2: decision and running max visible
    // ---------------- probabilities of tile t = i - kLag (if kept)
    const int t = i - kLag;
    const bool do_pv = (t >= 0) && dec[t % kDRing] != 0;
    if (do_pv) {
      const float* srow = s_ring + (t % kSRing) * G * kDecodeTile;
      for (int idx = tid; idx < G * kDecodeTile; idx += kDecThreads) {
        const int key = idx / G, r = idx % G;
        p_sm[idx] = ex2(srow[r * kDecodeTile + key] - m_sm[r]);
      }
    }
    // S3 (uniform): probabilities visible; also carries the V-wait give-up
    bool vok = true;
    if (do_pv)
      vok = mbar_wait(b_v_full(pv_count % kVStages), (pv_count / kVStages) & 1,
                      never, wait_limit_ns);
    if (__syncthreads_or(!vok)) {
      ok = false;
      break;
    }
    if (do_pv) {
      // move the reference max of this thread's partial sums if it changed
#pragma unroll
      for (int r = 0; r < G; ++r) {
        const float mn = m_sm[r];
        if (mn != m_used[r]) {
          const float a = ex2(m_used[r] - mn);
          lsum[r] *= a;
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[r][e] *= a;
          m_used[r] = mn;
        }
      }
      const uint8_t* vt = smem + C::kOffV + (pv_count % kVStages) * C::kTileBytes;
      const int key_lim = L - (t_begin + t) * kDecodeTile;
#pragma unroll
      for (int it = 0; it < C::kIters; ++it) {
        const int key = warp * (kDecodeTile / kWarps) + it * C::kKPI + sub;
        if (key < key_lim) {
          float vf[8];
          bf16x8_to_f32(*reinterpret_cast<const uint4*>(vt + key * D * 2 + c * 16), vf);
          float p[G];
#pragma unroll
          for (int r = 0; r < G; ++r) p[r] = p_sm[key * G + r];
#pragma unroll
          for (int r = 0; r < G; ++r) {
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[r][e] = fmaf(p[r], vf[e], acc[r][e]);
            if (c == 0) lsum[r] += p[r];
          }
        }
      }
      ++pv_count;
    }
  }

  if (!ok) {
    // leave no bulk copy in flight into this CTA's shared memory
    if (tid == 0) {
      atomicCAS(status, 0, ATTN_DEVICE_TIMEOUT_BASE + 20);
      for (int k = k_consumed; k < k_issued; ++k)
        mbar_drain(b_k_full(k % kKStages), (k / kKStages) & 1, wait_limit_ns);
      for (int k = pv_count; k < v_issued; ++k)
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
      for (int e = 0; e < 8; ++e) acc[r][e] += __shfl_xor_sync(0xffffffffu, acc[r][e], o);
    }
  }
  float* red = reinterpret_cast<float*>(smem + C::kOffK);  // [warp][G][D+1]
  __syncthreads();
  if (sub == 0) {
#pragma unroll
    for (int r = 0; r < G; ++r) {
#pragma unroll
      for (int e = 0; e < 8; ++e) red[(warp * G + r) * (D + 1) + c * 8 + e] = acc[r][e];
      if (c == 0) red[(warp * G + r) * (D + 1) + D] = lsum[r];
    }
  }
  __syncthreads();
  for (int idx = tid; idx < G * (D + 1); idx += kDecThreads) {
    const int r = idx / (D + 1), col = idx % (D + 1);
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) s += red[(w * G + r) * (D + 1) + col];
    red[(0 * G + r) * (D + 1) + col] = s;  // warp-0 slot is read below only after the sync
  }
  __syncthreads();
  for (int idx = tid; idx < G * D; idx += kDecThreads) {
    const int r = idx / D, col = idx % D;
    const float l = red[r * (D + 1) + D];
    const size_t row = static_cast<size_t>(b) * Hq + kv * G + r;
    o_part[(row * n_splits + split) * D + col] = red[r * (D + 1) + col] / l;
    // m_sm holds the reference max of the partial sums: skipped tiles never
    // move the running max, so it equals the value used by the last P*V
    if (col == 0) lse_part[row * n_splits + split] = m_sm[r] + __log2f(l);
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
