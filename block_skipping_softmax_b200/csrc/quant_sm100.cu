// 8-bit quantisation of Q or K for the low-precision Q K^T prefill paths.
// The int8 path follows "TurboAttention: Efficient Attention Approximation
// for High-Throughput LLM Serving" (Technical Deep Dive), which quantises Q
// and K to integers inside the FlashAttention tile loop.  No page names FP8:
// the e4m3 path is this library's own choice of a second 8-bit format on the
// same pipeline (the B200 tensor cores run e4m3 at the int8 rate).
//
// A tensor is cut into `groups` contiguous groups (one head slab [N, d] each
// for the prefill layouts).  Each group gets one power-of-two scale s, the
// smallest with max|x| <= M s, where M is the format's largest value (448
// for e4m3, 127 for int8), and every element becomes e4m3(x / s) or the
// integer nearest x / s, ties to even.  Because s is a power of two, x / s is
// exact, and the dequantised value code * s (three mantissa bits, or an
// integer of at most 7 bits) is exact in bf16: a bf16 reference fed the
// dequantised tensors sees exactly the operands the 8-bit MMAs see.
//
// Three launches, all bound by HBM: a per-group max of |x| (one atomic per
// block, on the bit pattern: non-negative floats order like their bits),
// the scale from the max, and the conversion.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "attn.h"

namespace bss {
int device_context(int* dev, int** status);  // api.cu
}

namespace {

constexpr int kThreads = 256;
constexpr int kVecPerThread = 4;                               // 16 elements each
constexpr long long kVecPerBlock = kThreads * kVecPerThread;   // 16 K elements per block

// |x| of 16 bf16 elements (one 32-byte vector), as the max of their bits.
__device__ __forceinline__ uint32_t absmax16(uint4 a, uint4 b) {
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    // bf16 -> fp32 is a 16-bit shift; clearing the sign gives |x|
    m = max(m, (w[i] << 16) & 0x7fffffffu);
    m = max(m, w[i] & 0x7fff0000u);
  }
  return m;
}

__global__ void __launch_bounds__(kThreads) amax_kernel(const uint4* __restrict__ x,
                                                        unsigned int* __restrict__ amax,
                                                        long long vec_per_group, long long blocks_per_group) {
  const long long g = blockIdx.x / blocks_per_group;
  const long long c = blockIdx.x % blocks_per_group;
  const uint4* src = x + 2 * g * vec_per_group;
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < kVecPerThread; ++i) {
    const long long v = c * kVecPerBlock + i * kThreads + threadIdx.x;
    if (v < vec_per_group) m = max(m, absmax16(src[2 * v], src[2 * v + 1]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ uint32_t wm[kThreads / 32];
  if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 1; i < kThreads / 32; ++i) m = max(m, wm[i]);
    if (m) atomicMax(amax + g, m);
  }
}

// In place: the max bits of each group become its scale.  max|x| = f 2^e with
// f in [0.5, 1), and M = m 2^p with m in [0.5, 1) (448 = 0.875 * 2^9,
// 127 = (127/128) * 2^7), so max|x| <= M 2^k holds first at k = e - p when
// f <= m, else at k = e - p + 1.  k is held at -126 or above, so that 1/s
// stays finite (only groups whose max is below about 2^-118 notice).  A zero
// group gets scale 1; a group holding inf or NaN gets NaN.
__global__ void scale_kernel(float* __restrict__ scales, long long groups, float m, int p) {
  const long long g = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (g >= groups) return;
  const uint32_t bits = __float_as_uint(scales[g]);
  float s;
  if (bits >= 0x7f800000u) {
    s = __uint_as_float(0x7fc00000u);
  } else if (bits == 0) {
    s = 1.f;
  } else {
    int e = 0;
    const float f = frexpf(__uint_as_float(bits), &e);
    s = ldexpf(1.f, max(f <= m ? e - p : e - p + 1, -126));
  }
  scales[g] = s;
}

template <bool INT8>
__global__ void __launch_bounds__(kThreads) convert_kernel(const uint4* __restrict__ x,
                                                           uint4* __restrict__ q,
                                                           const float* __restrict__ scales,
                                                           long long vec_per_group,
                                                           long long blocks_per_group) {
  const long long g = blockIdx.x / blocks_per_group;
  const long long c = blockIdx.x % blocks_per_group;
  const uint4* src = x + 2 * g * vec_per_group;
  uint4* dst = q + g * vec_per_group;
  const float inv = 1.f / __ldg(scales + g);  // a power of two: exact
#pragma unroll
  for (int i = 0; i < kVecPerThread; ++i) {
    const long long v = c * kVecPerBlock + i * kThreads + threadIdx.x;
    if (v >= vec_per_group) continue;
    const uint4 a = src[2 * v], b = src[2 * v + 1];
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t out[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      // elements 4k..4k+3 (low half of a word first) -> bytes 0..3 of out[k]
      const float e0 = __uint_as_float(w[2 * k] << 16) * inv;
      const float e1 = __uint_as_float(w[2 * k] & 0xffff0000u) * inv;
      const float e2 = __uint_as_float(w[2 * k + 1] << 16) * inv;
      const float e3 = __uint_as_float(w[2 * k + 1] & 0xffff0000u) * inv;
      if constexpr (INT8) {  // nearest integer, ties to even (|x / s| <= 127)
        const int i0 = __float2int_rn(e0), i1 = __float2int_rn(e1);
        const int i2 = __float2int_rn(e2), i3 = __float2int_rn(e3);
        out[k] = (static_cast<uint32_t>(i0) & 0xffu) | ((static_cast<uint32_t>(i1) & 0xffu) << 8) |
                 ((static_cast<uint32_t>(i2) & 0xffu) << 16) | (static_cast<uint32_t>(i3) << 24);
      } else {
        uint16_t lo, hi;  // cvt packs its first source into the upper byte
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(e1), "f"(e0));
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(e3), "f"(e2));
        out[k] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
      }
    }
    dst[v] = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int quantize(const void* x, void* q, float* scales, long long groups, long long group_elems,
             void* stream, bool int8) {
  if (!x || !q || !scales || groups <= 0 || group_elems <= 0) return ATTN_ERR_INVALID_ARG;
  if (group_elems % 16 != 0 || !aligned16(x) || !aligned16(q) ||
      (reinterpret_cast<uintptr_t>(scales) & 3u))
    return ATTN_ERR_INVALID_ARG;
  int dev = 0;
  int* status = nullptr;
  int st = bss::device_context(&dev, &status);
  if (st != ATTN_OK) return st;
  const long long vpg = group_elems / 16;
  const long long bpg = (vpg + kVecPerBlock - 1) / kVecPerBlock;
  if (groups > 0x7fffffffLL / bpg) return ATTN_ERR_UNSUPPORTED;
  const unsigned int grid = static_cast<unsigned int>(groups * bpg);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(scales, 0, static_cast<size_t>(groups) * sizeof(float), s) != cudaSuccess)
    return ATTN_ERR_CUDA;
  amax_kernel<<<grid, kThreads, 0, s>>>(static_cast<const uint4*>(x),
                                        reinterpret_cast<unsigned int*>(scales), vpg, bpg);
  const unsigned int sgrid = static_cast<unsigned int>((groups + 255) / 256);
  if (int8) {
    scale_kernel<<<sgrid, 256, 0, s>>>(scales, groups, 127.f / 128.f, 7);
    convert_kernel<true><<<grid, kThreads, 0, s>>>(static_cast<const uint4*>(x),
                                                   static_cast<uint4*>(q), scales, vpg, bpg);
  } else {
    scale_kernel<<<sgrid, 256, 0, s>>>(scales, groups, 0.875f, 9);
    convert_kernel<false><<<grid, kThreads, 0, s>>>(static_cast<const uint4*>(x),
                                                    static_cast<uint4*>(q), scales, vpg, bpg);
  }
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

extern "C" {

int attn_quantize_e4m3(const void* x, void* q, float* scales, long long groups,
                       long long group_elems, void* stream) {
  return quantize(x, q, scales, groups, group_elems, stream, false);
}

int attn_quantize_i8(const void* x, void* q, float* scales, long long groups,
                     long long group_elems, void* stream) {
  return quantize(x, q, scales, groups, group_elems, stream, true);
}

}  // extern "C"
