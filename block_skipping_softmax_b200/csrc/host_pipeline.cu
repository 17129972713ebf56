// Prefill from host memory: the batch is cut into chunks of KV-head groups
// (one KV head of one sequence with the g = Hq/Hkv query heads that read it;
// the groups of consecutive heads are consecutive in memory in every tensor)
// that flow through two device buffer sets on two streams, so the host-to-device
// copy of one chunk overlaps the kernel and the device-to-host copy of the
// previous one (PCIe copies run in both directions at once).  For a caller
// whose inputs live in (pinned) host memory this makes the whole call bound
// by the host-to-device copy instead of by the sum of copies and kernel.
//
// Host code only: every attention step runs in attn_prefill_ex's kernels.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "attn.h"

namespace {

constexpr int kMaxDevices = 64;
constexpr int kSets = 2;

struct HostPipe {
  cudaStream_t stream[kSets] = {nullptr, nullptr};
  cudaEvent_t start = nullptr;
  cudaEvent_t done[kSets] = {nullptr, nullptr};
  void* buf = nullptr;
  size_t bytes = 0;
};

std::mutex g_mu;  // one pipelined call at a time per process (the buffers are shared)
HostPipe g_pipe[kMaxDevices];

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

int ensure(HostPipe& p, size_t need) {
  for (int i = 0; i < kSets; ++i) {
    if (!p.stream[i] && cudaStreamCreateWithFlags(&p.stream[i], cudaStreamNonBlocking) != cudaSuccess)
      return ATTN_ERR_CUDA;
    if (!p.done[i] && cudaEventCreateWithFlags(&p.done[i], cudaEventDisableTiming) != cudaSuccess)
      return ATTN_ERR_CUDA;
  }
  if (!p.start && cudaEventCreateWithFlags(&p.start, cudaEventDisableTiming) != cudaSuccess)
    return ATTN_ERR_CUDA;
  if (p.bytes < need) {
    if (p.buf) {  // queued work of an earlier call may still use it
      cudaDeviceSynchronize();
      cudaFree(p.buf);
      p.buf = nullptr;
      p.bytes = 0;
    }
    if (cudaMalloc(&p.buf, need) != cudaSuccess) return ATTN_ERR_CUDA;
    p.bytes = need;
  }
  return ATTN_OK;
}

}  // namespace

extern "C" {

int attn_prefill_host(const void* Qh, const void* Kh, const void* Vh, void* Oh, int B, int Hq,
                      int Hkv, int N, int d, int causal, float tau, int Br, int Bc, int chunk,
                      void* stream) {
  if (!Qh || !Kh || !Vh || !Oh) return ATTN_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || N <= 0 || chunk < 0) return ATTN_ERR_INVALID_ARG;
  if (Hq % Hkv != 0 || (d != 64 && d != 128) || std::isnan(tau) || tau < 0.f)
    return ATTN_ERR_INVALID_ARG;
  if (!((Br == 64 && Bc == 64) || (Br == 128 && Bc == 64) || (Br == 128 && Bc == 128)))
    return ATTN_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
  // A chunk is `cb` KV-head groups.  Attention of one group touches nothing
  // outside it, so each chunk runs as a batch of cb "sequences" of g query
  // heads and one KV head, with the same per-row-block arithmetic (and bit
  // for bit the same output) as the whole batch on the device.
  const int g = Hq / Hkv;
  const long long n_groups_ll = static_cast<long long>(B) * Hkv;
  if (n_groups_ll > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  const int n_groups = static_cast<int>(n_groups_ll);
  const int cb = chunk > 0 ? (chunk < n_groups ? chunk : n_groups) : (n_groups + 7) / 8;
  const size_t q_seq = static_cast<size_t>(g) * N * d * 2;  // bytes of one group's Q (and O)
  const size_t kv_seq = static_cast<size_t>(N) * d * 2;     // of its K (and V)
  const size_t q_b = align256(q_seq * cb), kv_b = align256(kv_seq * cb);
  const size_t set_bytes = 2 * q_b + 2 * kv_b;  // Q, O, K, V
  std::lock_guard<std::mutex> lk(g_mu);
  HostPipe& p = g_pipe[dev];
  int st = ensure(p, kSets * set_bytes);
  if (st != ATTN_OK) return st;
  cudaStream_t caller = static_cast<cudaStream_t>(stream);
  if (cudaEventRecord(p.start, caller) != cudaSuccess) return ATTN_ERR_CUDA;
  for (int i = 0; i < kSets; ++i)
    if (cudaStreamWaitEvent(p.stream[i], p.start, 0) != cudaSuccess) return ATTN_ERR_CUDA;
  const char* qh = static_cast<const char*>(Qh);
  const char* kh = static_cast<const char*>(Kh);
  const char* vh = static_cast<const char*>(Vh);
  char* oh = static_cast<char*>(Oh);
  for (int c = 0, b0 = 0; b0 < n_groups; ++c, b0 += cb) {
    const int nb = (n_groups - b0 < cb) ? n_groups - b0 : cb;
    const int set = c % kSets;
    cudaStream_t s = p.stream[set];
    char* base = static_cast<char*>(p.buf) + set * set_bytes;
    char *qd = base, *od = base + q_b, *kd = base + 2 * q_b, *vd = base + 2 * q_b + kv_b;
    // a set's previous chunk ran on the same stream, so reusing it is ordered
    if (cudaMemcpyAsync(qd, qh + q_seq * b0, q_seq * nb, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(kd, kh + kv_seq * b0, kv_seq * nb, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(vd, vh + kv_seq * b0, kv_seq * nb, cudaMemcpyHostToDevice, s) != cudaSuccess)
      return ATTN_ERR_CUDA;
    st = attn_prefill_ex(qd, kd, vd, od, nb, g, 1, N, d, causal, tau, Br, Bc, s, nullptr);
    if (st != ATTN_OK) return st;
    if (cudaMemcpyAsync(oh + q_seq * b0, od, q_seq * nb, cudaMemcpyDeviceToHost, s) != cudaSuccess)
      return ATTN_ERR_CUDA;
  }
  for (int i = 0; i < kSets; ++i)
    if (cudaEventRecord(p.done[i], p.stream[i]) != cudaSuccess ||
        cudaStreamWaitEvent(caller, p.done[i], 0) != cudaSuccess)
      return ATTN_ERR_CUDA;
  return ATTN_OK;
}

}  // extern "C"

namespace bss {

// Frees the pipeline's buffers, streams and events (called by attn_shutdown).
void host_pipeline_release() {
  std::lock_guard<std::mutex> lk(g_mu);
  int cur = 0;
  const bool have = cudaGetDevice(&cur) == cudaSuccess;
  for (int dev = 0; dev < kMaxDevices; ++dev) {
    HostPipe& p = g_pipe[dev];
    if (!p.buf && !p.start) continue;
    if (cudaSetDevice(dev) != cudaSuccess) continue;
    cudaDeviceSynchronize();
    if (p.buf) cudaFree(p.buf);
    for (int i = 0; i < kSets; ++i) {
      if (p.stream[i]) cudaStreamDestroy(p.stream[i]);
      if (p.done[i]) cudaEventDestroy(p.done[i]);
    }
    if (p.start) cudaEventDestroy(p.start);
    p = HostPipe{};
  }
  if (have) cudaSetDevice(cur);
}

}  // namespace bss
