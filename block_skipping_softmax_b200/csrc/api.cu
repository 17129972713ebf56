// C ABI of libattn.so: argument validation, device checks, workspace and the
// device status word.  Every compute step runs in the kernels; this layer only
// checks arguments, encodes TMA descriptors (in the launchers) and launches.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "attn.h"
#include "kernels.cuh"

namespace {

__device__ int g_status;  // 0, or ATTN_DEVICE_TIMEOUT_BASE + site of a wait that gave up

constexpr int kMaxDevices = 64;
constexpr float kLog2e = 1.4426950408889634f;

std::mutex g_mu;
cudaStream_t g_stream = nullptr;
unsigned long long g_wait_limit_ns = 2000ull * 1000ull * 1000ull;
int g_last_site = 0;
int g_withhold_v = 0;  // test support, see attn_test_withhold_copy
int g_dev_checked[kMaxDevices];  // 0 unknown, 1 sm_100, 2 other
int* g_status_ptr[kMaxDevices];
void* g_ws[kMaxDevices];
size_t g_ws_bytes[kMaxDevices];

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device check and per-device status word; returns ATTN_OK or an error.
int device_ready(int* dev_out, int** status_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_UNSUPPORTED;
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_dev_checked[dev] == 0) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return ATTN_ERR_CUDA;
    g_dev_checked[dev] = (prop.major == 10 && prop.minor == 0) ? 1 : 2;
    if (g_dev_checked[dev] == 1) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) {
        g_dev_checked[dev] = 0;
        return ATTN_ERR_CUDA;
      }
      g_status_ptr[dev] = static_cast<int*>(p);
    }
  }
  if (g_dev_checked[dev] != 1) return ATTN_ERR_UNSUPPORTED;
  *dev_out = dev;
  *status_out = g_status_ptr[dev];
  return ATTN_OK;
}

bool tau_ok(float tau) { return !std::isnan(tau) && tau >= 0.f; }

int check_prefill(const void* Q, const void* K, const void* V, const void* O, int B, int Hq,
                  int Hkv, int N, int d, float tau, int Br, int Bc) {
  if (!Q || !K || !V || !O) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return ATTN_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || N <= 0) return ATTN_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_INVALID_ARG;
  if (!((Br == 64 && Bc == 64) || (Br == 128 && Bc == 64) || (Br == 128 && Bc == 128)))
    return ATTN_ERR_INVALID_ARG;
  if (!tau_ok(tau)) return ATTN_ERR_INVALID_ARG;
  const long long n_rb = (N + Br - 1) / Br;
  if (n_rb * B * Hq > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  return ATTN_OK;
}

int check_decode(const void* q, const void* K, const void* V, const void* o, int B, int Hq,
                 int Hkv, int L, int d, float tau) {
  if (!q || !K || !V || !o) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(K) || !aligned16(V) || !aligned16(o)) return ATTN_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || L <= 0) return ATTN_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_INVALID_ARG;
  if (!tau_ok(tau)) return ATTN_ERR_INVALID_ARG;
  const int g = Hq / Hkv;
  if (g != 1 && g != 2 && g != 4 && g != 8) return ATTN_ERR_UNSUPPORTED;
  if (Hkv > 65535 || B > 65535) return ATTN_ERR_UNSUPPORTED;
  return ATTN_OK;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

void decode_ws_layout(int B, int Hq, int n_splits, int d, size_t* o_bytes, size_t* total) {
  *o_bytes = align256(static_cast<size_t>(B) * Hq * n_splits * d * sizeof(float));
  *total = *o_bytes + align256(static_cast<size_t>(B) * Hq * n_splits * sizeof(float));
}

}  // namespace

namespace bss {
void host_pipeline_release();  // host_pipeline.cu
// Current device (sm_100 checked) and its device status word, for entry
// points defined in other files.
int device_context(int* dev, int** status) { return device_ready(dev, status); }
unsigned long long wait_limit_ns() { return g_wait_limit_ns; }
// The decode argument checks, for decode entry points defined in other files.
int check_decode_args(const void* q, const void* K, const void* V, const void* o, int B, int Hq,
                      int Hkv, int L, int d, float tau) {
  return check_decode(q, K, V, o, B, Hq, Hkv, L, d, tau);
}
}  // namespace bss

extern "C" {

int attn_prefill_ex(const void* Q, const void* K, const void* V, void* O, int B, int Hq, int Hkv,
                    int N, int d, int causal, float tau, int Br, int Bc, void* stream,
                    uint8_t* skip_mask) {
  int st = check_prefill(Q, K, V, O, B, Hq, Hkv, N, d, tau, Br, Bc);
  if (st != ATTN_OK) return st;
  int dev = 0;
  int* status = nullptr;
  if ((st = device_ready(&dev, &status)) != ATTN_OK) return st;
  bss::PrefillLaunch a{};
  a.Q = Q;
  a.K = K;
  a.V = V;
  a.O = O;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.N = N;
  a.d = d;
  a.causal = causal ? 1 : 0;
  a.Br = Br;
  a.Bc = Bc;
  a.scale_log2 = kLog2e / std::sqrt(static_cast<float>(d));
  a.tau_is_inf = std::isinf(tau) ? 1 : 0;
  a.tau_log2 = a.tau_is_inf ? 0.f : tau * kLog2e;
  a.skip_mask = skip_mask;
  a.status = status;
  a.wait_limit_ns = g_wait_limit_ns;
  a.stream = static_cast<cudaStream_t>(stream);
  return Br == 128 ? bss::launch_prefill_pp(a) : bss::launch_prefill(a);
}

int attn_prefill_poly(const void* Q, const void* K, const void* V, void* O, int B, int Hq,
                      int Hkv, int N, int d, int causal, float tau, int Br, int Bc, int poly_pairs,
                      void* stream, uint8_t* skip_mask) {
  if (poly_pairs != 0 && poly_pairs != 4 && poly_pairs != 8) return ATTN_ERR_INVALID_ARG;
  if (d != 128 || Br != 128 || Bc != 128) return ATTN_ERR_INVALID_ARG;
  int st = check_prefill(Q, K, V, O, B, Hq, Hkv, N, d, tau, Br, Bc);
  if (st != ATTN_OK) return st;
  int dev = 0;
  int* status = nullptr;
  if ((st = device_ready(&dev, &status)) != ATTN_OK) return st;
  bss::PrefillLaunch a{};
  a.Q = Q;
  a.K = K;
  a.V = V;
  a.O = O;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.N = N;
  a.d = d;
  a.causal = causal ? 1 : 0;
  a.Br = Br;
  a.Bc = Bc;
  a.scale_log2 = kLog2e / std::sqrt(static_cast<float>(d));
  a.tau_is_inf = std::isinf(tau) ? 1 : 0;
  a.tau_log2 = a.tau_is_inf ? 0.f : tau * kLog2e;
  a.skip_mask = skip_mask;
  a.status = status;
  a.wait_limit_ns = g_wait_limit_ns;
  a.stream = static_cast<cudaStream_t>(stream);
  a.poly_pairs = poly_pairs;
  return bss::launch_prefill_split(a);
}

int attn_prefill_varlen(const void* Q, const void* K, const void* V, void* O,
                        const int32_t* cu_seqlens, int B, int max_seqlen, int total_tokens, int Hq,
                        int Hkv, int d, int causal, float tau, int Br, int Bc, void* stream,
                        uint8_t* skip_mask) {
  if (!cu_seqlens || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)) return ATTN_ERR_INVALID_ARG;
  if (total_tokens <= 0 || max_seqlen <= 0) return ATTN_ERR_INVALID_ARG;
  if (Br != 128) return ATTN_ERR_INVALID_ARG;  // the persistent two-row-block kernel only
  int st = check_prefill(Q, K, V, O, B, Hq, Hkv, max_seqlen, d, tau, Br, Bc);
  if (st != ATTN_OK) return st;
  int dev = 0;
  int* status = nullptr;
  if ((st = device_ready(&dev, &status)) != ATTN_OK) return st;
  bss::PrefillLaunch a{};
  a.Q = Q;
  a.K = K;
  a.V = V;
  a.O = O;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.N = max_seqlen;
  a.d = d;
  a.causal = causal ? 1 : 0;
  a.Br = Br;
  a.Bc = Bc;
  a.scale_log2 = kLog2e / std::sqrt(static_cast<float>(d));
  a.tau_is_inf = std::isinf(tau) ? 1 : 0;
  a.tau_log2 = a.tau_is_inf ? 0.f : tau * kLog2e;
  a.skip_mask = skip_mask;
  a.status = status;
  a.wait_limit_ns = g_wait_limit_ns;
  a.stream = static_cast<cudaStream_t>(stream);
  a.cu_seqlens = cu_seqlens;
  a.total = total_tokens;
  return bss::launch_prefill_pp(a);
}

static int prefill_8bit(const void* Q8, const void* K8, const float* q_scales, const float* k_scales,
                        const void* V, void* O, int B, int Hq, int Hkv, int N, int d, int causal, float tau,
                        int Br, int Bc, void* stream, uint8_t* skip_mask, int format) {
  if (!q_scales || !k_scales) return ATTN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(q_scales) & 3u) || (reinterpret_cast<uintptr_t>(k_scales) & 3u))
    return ATTN_ERR_INVALID_ARG;
  if (d != 128 || Br != 128) return ATTN_ERR_INVALID_ARG;
  int st = check_prefill(Q8, K8, V, O, B, Hq, Hkv, N, d, tau, Br, Bc);
  if (st != ATTN_OK) return st;
  int dev = 0;
  int* status = nullptr;
  if ((st = device_ready(&dev, &status)) != ATTN_OK) return st;
  bss::PrefillLaunch a{};
  a.Q = Q8;
  a.K = K8;
  a.V = V;
  a.O = O;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.N = N;
  a.d = d;
  a.causal = causal ? 1 : 0;
  a.Br = Br;
  a.Bc = Bc;
  a.scale_log2 = kLog2e / std::sqrt(static_cast<float>(d));
  a.tau_is_inf = std::isinf(tau) ? 1 : 0;
  a.tau_log2 = a.tau_is_inf ? 0.f : tau * kLog2e;
  a.skip_mask = skip_mask;
  a.status = status;
  a.wait_limit_ns = g_wait_limit_ns;
  a.stream = static_cast<cudaStream_t>(stream);
  a.q_scales = q_scales;
  a.k_scales = k_scales;
  a.qk_format = format;
  return bss::launch_prefill_pp(a);
}

int attn_prefill_qk8(const void* Q8, const void* K8, const float* q_scales, const float* k_scales,
                     const void* V, void* O, int B, int Hq, int Hkv, int N, int d, int causal,
                     float tau, int Br, int Bc, void* stream, uint8_t* skip_mask) {
  return prefill_8bit(Q8, K8, q_scales, k_scales, V, O, B, Hq, Hkv, N, d, causal, tau, Br, Bc, stream,
                      skip_mask, 1);
}

int attn_prefill_qki8(const void* Q8, const void* K8, const float* q_scales, const float* k_scales,
                      const void* V, void* O, int B, int Hq, int Hkv, int N, int d, int causal,
                      float tau, int Br, int Bc, void* stream, uint8_t* skip_mask) {
  return prefill_8bit(Q8, K8, q_scales, k_scales, V, O, B, Hq, Hkv, N, d, causal, tau, Br, Bc, stream,
                      skip_mask, 2);
}

int attn_prefill(const void* Q, const void* K, const void* V, void* O, int B, int Hq, int Hkv,
                 int N, int d, int causal, float tau, int Br, int Bc) {
  return attn_prefill_ex(Q, K, V, O, B, Hq, Hkv, N, d, causal, tau, Br, Bc, g_stream, nullptr);
}

int attn_decode_tile(void) { return bss::kDecodeTile; }

int attn_decode_split_len(int B, int Hkv, int L) {
  if (B <= 0 || Hkv <= 0 || L <= 0) return -1;
  // Choose tiles-per-split to minimise modelled time: waves of 296 resident
  // CTAs (148 SMs x 2) times (tiles per CTA + ~2 tiles of start-up cost).
  const long long slots = 296;
  const long long groups = static_cast<long long>(B) * Hkv;
  const long long n_tiles = (L + bss::kDecodeTile - 1) / bss::kDecodeTile;
  // A split's running max starts at -inf, so its first tile is always kept:
  // splits are at least 8 tiles (512 keys) long so that the skip test has a
  // history to compare against.
  const long long min_tps = n_tiles < 8 ? n_tiles : 8;
  long long best_tps = n_tiles, best_cost = -1;
  for (long long tps = n_tiles; tps >= min_tps; --tps) {
    const long long ns = (n_tiles + tps - 1) / tps;
    if (ns > 4096) break;
    const long long waves = (groups * ns + slots - 1) / slots;
    const long long cost = waves * (tps + 2);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best_tps = tps;
    }
  }
  return static_cast<int>(best_tps * bss::kDecodeTile);
}

size_t attn_decode_workspace_bytes(int B, int Hq, int Hkv, int L, int d) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || L <= 0 || (d != 64 && d != 128)) return 0;
  const int ls = attn_decode_split_len(B, Hkv, L);
  const int n_splits = (L + ls - 1) / ls;
  size_t ob = 0, total = 0;
  decode_ws_layout(B, Hq, n_splits, d, &ob, &total);
  return total;
}

int attn_decode_ex(const void* q, const void* K, const void* V, void* o, int B, int Hq, int Hkv,
                   int L, int d, float tau, void* stream, uint8_t* skip_mask, void* ws,
                   size_t ws_bytes) {
  return attn_decode_rule(q, K, V, o, B, Hq, Hkv, L, d, tau, ATTN_DECODE_RULE_GROUP, stream,
                          skip_mask, ws, ws_bytes);
}

}  // extern "C"

namespace {

// Shared tail of the decode entry points: split layout, workspace, launch.
int run_decode(bss::DecodeLaunch& a, int dev, void* ws, size_t ws_bytes) {
  const int ls = attn_decode_split_len(a.B, a.Hkv, a.L);
  const int n_splits = (a.L + ls - 1) / ls;
  size_t ob = 0, need = 0;
  decode_ws_layout(a.B, a.Hq, n_splits, a.d, &ob, &need);
  if (ws == nullptr) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_ws_bytes[dev] < need) {
      // the old buffer may still be read by queued work on another stream
      if (g_ws[dev]) {
        cudaDeviceSynchronize();
        cudaFree(g_ws[dev]);
        g_ws[dev] = nullptr;
        g_ws_bytes[dev] = 0;
      }
      if (cudaMalloc(&g_ws[dev], need) != cudaSuccess) return ATTN_ERR_CUDA;
      g_ws_bytes[dev] = need;
    }
    ws = g_ws[dev];
  } else if (ws_bytes < need) {
    return ATTN_ERR_INVALID_ARG;
  }
  a.scale_log2 = kLog2e / std::sqrt(static_cast<float>(a.d));
  a.split_len = ls;
  a.n_splits = n_splits;
  a.o_part = static_cast<float*>(ws);
  a.lse_part = reinterpret_cast<float*>(static_cast<char*>(ws) + ob);
  a.wait_limit_ns = g_wait_limit_ns;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    a.withhold_v = g_withhold_v;
  }
  return bss::launch_decode(a);
}

bool rule_ok(int rule) { return (rule & ~(ATTN_DECODE_RULE_PER_HEAD | ATTN_DECODE_RULE_SINK_SEED)) == 0; }

}  // namespace

extern "C" {

int attn_decode_rule(const void* q, const void* K, const void* V, void* o, int B, int Hq, int Hkv,
                     int L, int d, float tau, int rule, void* stream, uint8_t* skip_mask, void* ws,
                     size_t ws_bytes) {
  if (!rule_ok(rule)) return ATTN_ERR_INVALID_ARG;
  int st = check_decode(q, K, V, o, B, Hq, Hkv, L, d, tau);
  if (st != ATTN_OK) return st;
  if (ws == nullptr && ws_bytes != 0) return ATTN_ERR_INVALID_ARG;
  if (ws != nullptr && (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return ATTN_ERR_INVALID_ARG;
  int dev = 0;
  int* status = nullptr;
  if ((st = device_ready(&dev, &status)) != ATTN_OK) return st;
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
  a.tau_is_inf = std::isinf(tau) ? 1 : 0;
  a.tau_log2 = a.tau_is_inf ? 0.f : tau * kLog2e;
  a.skip_mask = skip_mask;
  a.status = status;
  a.stream = static_cast<cudaStream_t>(stream);
  a.rule = rule;
  return run_decode(a, dev, ws, ws_bytes);
}

int attn_decode_paged(const void* q, const void* K_pages, const void* V_pages,
                      const int32_t* block_table, const int32_t* seq_lens, void* o, int B, int Hq,
                      int Hkv, int num_pages, int max_pages_per_seq, int max_seq_len, int d,
                      float tau, int rule, void* stream, uint8_t* skip_mask, void* ws,
                      size_t ws_bytes) {
  if (!rule_ok(rule)) return ATTN_ERR_INVALID_ARG;
  if (!block_table || !seq_lens) return ATTN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(block_table) & 3u) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
    return ATTN_ERR_INVALID_ARG;
  if (num_pages <= 0 || max_pages_per_seq <= 0) return ATTN_ERR_INVALID_ARG;
  if (static_cast<long long>(num_pages) * Hkv > (1ll << 31) - 1) return ATTN_ERR_UNSUPPORTED;
  if (max_seq_len > static_cast<long long>(max_pages_per_seq) * bss::kDecodeTile)
    return ATTN_ERR_INVALID_ARG;
  int st = check_decode(q, K_pages, V_pages, o, B, Hq, Hkv, max_seq_len, d, tau);
  if (st != ATTN_OK) return st;
  if (ws == nullptr && ws_bytes != 0) return ATTN_ERR_INVALID_ARG;
  if (ws != nullptr && (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return ATTN_ERR_INVALID_ARG;
  int dev = 0;
  int* status = nullptr;
  if ((st = device_ready(&dev, &status)) != ATTN_OK) return st;
  bss::DecodeLaunch a{};
  a.q = q;
  a.K = K_pages;
  a.V = V_pages;
  a.o = o;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.L = max_seq_len;
  a.d = d;
  a.tau_is_inf = std::isinf(tau) ? 1 : 0;
  a.tau_log2 = a.tau_is_inf ? 0.f : tau * kLog2e;
  a.skip_mask = skip_mask;
  a.status = status;
  a.stream = static_cast<cudaStream_t>(stream);
  a.rule = rule;
  a.block_table = block_table;
  a.seq_lens = seq_lens;
  a.max_pages = max_pages_per_seq;
  a.num_pages = num_pages;
  return run_decode(a, dev, ws, ws_bytes);
}

int attn_decode(const void* q, const void* K, const void* V, void* o, int B, int Hq, int Hkv,
                int L, int d, float tau) {
  return attn_decode_ex(q, K, V, o, B, Hq, Hkv, L, d, tau, g_stream, nullptr, nullptr, 0);
}

int attn_set_stream(void* stream) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_stream = static_cast<cudaStream_t>(stream);
  return ATTN_OK;
}

int attn_set_wait_limit_ms(int ms) {
  if (ms < 1) return ATTN_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_mu);
  g_wait_limit_ns = static_cast<unsigned long long>(ms) * 1000000ull;
  return ATTN_OK;
}

int attn_test_withhold_copy(int which) {
  if (which != 0 && which != 1) return ATTN_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_mu);
  g_withhold_v = which;
  return ATTN_OK;
}

int attn_sync_status(void) {
  int dev = 0;
  int* status = nullptr;
  int st = device_ready(&dev, &status);
  if (st != ATTN_OK) return st;
  if (cudaDeviceSynchronize() != cudaSuccess) return ATTN_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    g_last_site = v - ATTN_DEVICE_TIMEOUT_BASE;
    return ATTN_ERR_TIMEOUT;
  }
  return ATTN_OK;
}

int attn_last_timeout_site(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  return g_last_site;
}

const char* attn_status_string(int s) {
  switch (s) {
    case ATTN_OK: return "ATTN_OK";
    case ATTN_ERR_INVALID_ARG: return "ATTN_ERR_INVALID_ARG";
    case ATTN_ERR_UNSUPPORTED: return "ATTN_ERR_UNSUPPORTED";
    case ATTN_ERR_CUDA: return "ATTN_ERR_CUDA";
    case ATTN_ERR_TIMEOUT: return "ATTN_ERR_TIMEOUT";
    default: return "ATTN_ERR_UNKNOWN";
  }
}

void attn_shutdown(void) {
  bss::host_pipeline_release();
  std::lock_guard<std::mutex> lk(g_mu);
  int cur = 0;
  const bool have = cudaGetDevice(&cur) == cudaSuccess;
  for (int dev = 0; dev < kMaxDevices; ++dev) {
    if (!g_ws[dev]) continue;
    if (cudaSetDevice(dev) == cudaSuccess) {
      cudaDeviceSynchronize();
      cudaFree(g_ws[dev]);
    }
    g_ws[dev] = nullptr;
    g_ws_bytes[dev] = 0;
  }
  if (have) cudaSetDevice(cur);
}

}  // extern "C"
