// Host-side internals shared by the translation units of libpagedkv.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/pagedkv.h"

namespace pkv {

// Records a message for pkv_last_error() and returns `status`.
int fail(int status, const char* fmt, ...);

// Clears the message pkv_last_error() returns (at the start of each entry point).
void clear_last_error();

// SM count of the current device (cached per device).
int device_sm_count();

// Returns PKV_OK, or PKV_ERR_CUDA after recording cudaGetLastError().
int check_launch(const char* what);

// Argument checks shared by the entry points (record a message, return a status).
int check_cache(const pkv_cache_desc& c, const char* fn);
int check_mask(const pkv_mask_mod& m, const char* fn);
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

inline int dtype_size(int32_t dt) { return dt == PKV_BF16 ? 2 : dt == PKV_FP8_E4M3 ? 1 : 4; }

inline int log2_int(int32_t x) {
  int r = 0;
  while ((1 << r) < x) ++r;
  return r;
}

int launch_append(const void* k, const void* v, const int64_t* slots, int32_t num_tokens,
                  void* k_cache, void* v_cache, const pkv_cache_desc& c, int32_t* dbg,
                  cudaStream_t s);

// bf16 tokens quantised into E4M3 pools with a float32 scale per stored row.
int launch_append_fp8(const void* k, const void* v, const int64_t* slots, int32_t num_tokens,
                      void* k_cache, void* v_cache, float* k_scale, float* v_scale,
                      const pkv_cache_desc& c, int32_t* dbg, cudaStream_t s);

int launch_gather(const void* k_cache, const void* v_cache, const pkv_cache_desc& c,
                  const int32_t* tables, int32_t max_blocks, const int32_t* lens, int32_t batch,
                  int32_t out_max_len, void* k_out, void* v_out, int32_t* dbg, cudaStream_t s);

// With skip_unset, pairs (-1, -1) copy nothing (a list with holes).
// Copies num_pairs (src, dst) spans of bytes_per_block (a multiple of 16)
// bytes in two arrays of num_blocks spans each (pools, or their row scales).
int launch_copy_spans(void* a, void* b, int64_t bytes_per_block, int32_t num_blocks,
                      const int32_t* pairs, int32_t num_pairs, int32_t* dbg, cudaStream_t s,
                      bool skip_unset = false);
int launch_copy_blocks(void* k_cache, void* v_cache, const pkv_cache_desc& c,
                       const int32_t* pairs, int32_t num_pairs, int32_t* dbg, cudaStream_t s,
                       bool skip_unset = false);

struct DecodeArgs {
  const void* q;
  const void* k_cache;
  const void* v_cache;
  pkv_cache_desc cache;
  const int32_t* tables;
  int32_t max_blocks;
  const int32_t* seq_lens;
  int32_t batch;
  int32_t num_q_heads;
  float scale;
  pkv_mask_mod mask;
  void* out;
  float* lse;
  void* workspace;
  size_t workspace_bytes;
  int32_t* dbg;
  cudaStream_t stream;
  const float* k_scale = nullptr;  // E4M3 pools: row scales [num_blocks * Hkv * block_size]
  const float* v_scale = nullptr;
  // fused append (bf16 pools): newest token of each sequence [batch, Hkv, head_dim]
  const void* k_new = nullptr;
  const void* v_new = nullptr;
};

size_t decode_workspace_size(int32_t batch, int32_t num_q_heads, const pkv_cache_desc& c);
int launch_decode(const DecodeArgs& a);

struct PrefillArgs {
  const void* q;
  const void* k_new;
  const void* v_new;
  const void* k_cache;
  const void* v_cache;
  pkv_cache_desc cache;
  const int32_t* tables;
  int32_t max_blocks;
  const int32_t* ctx_lens;
  const int32_t* q_lens;
  int32_t batch;
  int32_t total_q;
  int32_t num_q_heads;
  float scale;
  pkv_mask_mod mask;
  void* out;
  float* lse;
  int32_t* dbg;
  cudaStream_t stream;
};

int launch_prefill(const PrefillArgs& a);


// Encodes a 2-D bf16 tensor map over a pool viewed as [rows, head_dim] with a
// [box_rows, 64]-element box and 128-byte swizzle. Returns false on failure.
bool make_pool_tensor_map(void* map_out, const void* base, int64_t rows, int32_t head_dim,
                          int32_t box_rows);

// Same over a pool of one-byte codes, box [box_rows, 128] (128-byte swizzle).
bool make_pool_tensor_map_u8(void* map_out, const void* base, int64_t rows, int32_t head_dim,
                             int32_t box_rows);

// Encodes a bf16 tensor map of rank 1..5 with 128-byte swizzle; dims and
// box innermost first, strides in bytes for dims 1..rank-1.
bool make_tensor_map_bf16(void* map_out, const void* base, int rank, const uint64_t* dims,
                          const uint64_t* strides_bytes, const uint32_t* box);

}  // namespace pkv
