// Internal launch descriptors shared by the C-ABI layer and the kernels.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <cstddef>
#include <cstdint>

#include "attn.h"

namespace bss {

struct PrefillLaunch {
  const void* Q;
  const void* K;
  const void* V;
  void* O;
  int B, Hq, Hkv, N, d, causal, Br, Bc;
  float scale_log2;  // log2(e) / sqrt(d): scores in log2 units
  float tau_log2;    // tau * log2(e)
  int tau_is_inf;
  uint8_t* skip_mask;
  int* status;
  unsigned long long wait_limit_ns;
  cudaStream_t stream;
  // variable-length batch (cu_seqlens != nullptr): Q, O [total, Hq, d] and
  // K, V [total, Hkv, d]; sequence b is tokens [cu_seqlens[b], cu_seqlens[b+1])
  // and N is the longest sequence
  const int* cu_seqlens;
  int total;
  // e4m3 Q and K (q_scales != nullptr): Q [B, Hq, N, d] and K [B, Hkv, N, d]
  // hold one byte per element, head slab (b, h) scaled by q_scales[b*Hq+h]
  // (k_scales[b*Hkv+h]); V and O stay bf16
  const float* q_scales;
  const float* k_scales;
  int qk_format;  // with q_scales: 1 e4m3, 2 signed int8
  // exponential pairs (of every 16) computed by the FMA-pipe polynomial
  // instead of MUFU: 0, 4 or 8 (column-split kernel, d = Bc = 128)
  int poly_pairs;
};

int launch_prefill(const PrefillLaunch& a);     // one row block per CTA (any Br)
int launch_prefill_pp(const PrefillLaunch& a);  // two row blocks per CTA, Br = 128
// one row block per work item, the softmax warpgroups splitting each key
// tile's columns: d = 128, Br = 128, fixed-length bf16 batches
int launch_prefill_split(const PrefillLaunch& a);

// Tensor map over [BH, rows, D] bf16 (d fastest): boxes of 64 columns x
// box_rows rows, 128-byte swizzle; rows past `rows` read as zeros.
bool tma_map_bhnd(CUtensorMap* m, const void* base, int BH, int rows, int D, int box_rows);

constexpr int kDecodeTile = 64;  // keys per decode tile

struct DecodeLaunch {
  const void* q;
  const void* K;
  const void* V;
  void* o;
  int B, Hq, Hkv, L, d;
  float scale_log2;
  float tau_log2;
  int tau_is_inf;
  int split_len;  // keys per split, multiple of kDecodeTile
  int n_splits;
  float* o_part;    // [B*Hq, n_splits, d] fp32 (normalised partial outputs)
  float* lse_part;  // [B*Hq, n_splits]    fp32 (log2-sum-exp of each split)
  uint8_t* skip_mask;
  int* status;
  unsigned long long wait_limit_ns;
  cudaStream_t stream;
  int withhold_v;  // test support: 1 = every CTA withholds its first V copy
  int rule;        // ATTN_DECODE_RULE_* bits
  // paged KV cache (block_table == nullptr: contiguous [B, Hkv, L, d]); then
  // K and V are page pools [num_pages, Hkv, 64, d] and L is the longest
  // sequence
  const int* block_table;  // [B, max_pages] page ids
  const int* seq_lens;     // [B] keys per sequence
  int max_pages;
  int num_pages;
};

int launch_decode(const DecodeLaunch& a);

}  // namespace bss
