// Decode for callers that cannot allocate device memory.
//
// Split-KV decode needs scratch space for its per-split partial results.
// attn_decode gets it with cudaMalloc (on its first call, and again whenever
// a larger problem arrives) and attn_decode_ex asks the caller for a buffer.
// Some callers can do neither: a serving engine that reserves nearly all of
// HBM up front for its own KV-cache pool and accounts for every byte (a
// library allocation there can fail, or eat memory the engine promised to
// someone else), a latency-critical loop that cannot afford the device-wide
// synchronisation that cudaMalloc/cudaFree may imply, or a host that talks to
// this library through a minimal binding that only passes q, K, V and o.
//
// For them, attn_decode_noalloc keeps the scratch in the fixed array below, in
// device global memory.  It is reserved on every GPU that loads this library
// and held until the process exits.  Nothing here calls cudaMalloc, cudaFree
// or any allocating library routine.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "attn.h"
#include "kernels.cuh"

namespace bss {
int device_context(int* dev, int** status);  // defined in api.cu
unsigned long long wait_limit_ns();          // defined in api.cu
int check_decode_args(const void* q, const void* K, const void* V, const void* o, int B, int Hq,
                      int Hkv, int L, int d, float tau);  // defined in api.cu
}

namespace {

constexpr size_t kScratchBytes = size_t(16) << 20;  // 16 MiB per GPU
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices];  // device address of g_decode_scratch, per device

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Once per device, with that device current: the device address of the array.
// In host code the array's name is only a host-side stand-in; a kernel must be
// given this address instead.
int scratch_address(int dev, void** out) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr)
      return ATTN_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return ATTN_OK;
}

}  // namespace

extern "C" int attn_decode_noalloc(const void* q, const void* K, const void* V, void* o, int B,
                                   int Hq, int Hkv, int L, int d, float tau, void* stream,
                                   uint8_t* skip_mask) {
  // the same argument checks as attn_decode_ex, before any CUDA call
  int st = bss::check_decode_args(q, K, V, o, B, Hq, Hkv, L, d, tau);
  if (st != ATTN_OK) return st;

  // same split layout as attn_decode, so results are identical
  const int ls = attn_decode_split_len(B, Hkv, L);
  const int n_splits = (L + ls - 1) / ls;
  const size_t o_bytes = round256(static_cast<size_t>(B) * Hq * n_splits * d * sizeof(float));
  const size_t need = o_bytes + round256(static_cast<size_t>(B) * Hq * n_splits * sizeof(float));
  if (need > kScratchBytes) return ATTN_ERR_UNSUPPORTED;  // problem too large for the array

  int dev = 0;
  int* status = nullptr;
  st = bss::device_context(&dev, &status);
  if (st != ATTN_OK) return st;
  void* scratch = nullptr;
  if ((st = scratch_address(dev, &scratch)) != ATTN_OK) return st;

  // Every scratch entry the combine kernel reads is written earlier in the
  // same call by the partial kernel (a CTA whose bounded wait gives up writes
  // its split as empty), so nothing needs clearing.
  bss::DecodeLaunch a{};
  a.q = q;
  a.K = K;
  a.V = V;
  a.o = o;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.L = L;
  a.d = d;
  a.scale_log2 = 1.4426950408889634f / std::sqrt(static_cast<float>(d));
  a.tau_is_inf = std::isinf(tau) ? 1 : 0;
  a.tau_log2 = a.tau_is_inf ? 0.f : tau * 1.4426950408889634f;
  a.split_len = ls;
  a.n_splits = n_splits;
  a.o_part = static_cast<float*>(scratch);
  a.lse_part = reinterpret_cast<float*>(static_cast<char*>(scratch) + o_bytes);
  a.skip_mask = skip_mask;
  a.status = status;
  a.wait_limit_ns = bss::wait_limit_ns();
  a.stream = static_cast<cudaStream_t>(stream);
  return bss::launch_decode(a);
}
