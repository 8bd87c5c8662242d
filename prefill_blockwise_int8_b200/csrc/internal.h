// Internal launch interface between the C ABI (tilemix_api.cu) and the
// kernels.  Not installed, not part of the ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace tilemix {

// Device-side status codes (same values as tilemix_status).
constexpr int kStatusTimeout = 4;
constexpr int kStatusBadSeqlens = 5;

// Stores `code` into *status if the word is still 0.
__device__ __forceinline__ void report_status(int32_t* status, int code) {
  if (status) atomicCAS(reinterpret_cast<int*>(status), 0, code);
}

cudaError_t launch_quantize_blockwise(const void* x, const int32_t* cu_seqlens,
                                      int batch, int max_seqlen,
                                      int total_tokens, int heads,
                                      int head_dim, int block, int8_t* x8,
                                      float* scale, int32_t* status,
                                      cudaStream_t stream);

// Q and K in one launch (the same results as one launch each).
cudaError_t launch_quantize_blockwise_qk(
    const void* q, const void* k, const int32_t* cu_seqlens, int batch,
    int max_seqlen, int total_tokens, int hq, int hkv, int head_dim,
    int block_q, int block_k, int8_t* q8, float* q_scale, int8_t* k8,
    float* k_scale, int32_t* status, cudaStream_t stream);

cudaError_t launch_pack_mask(const uint8_t* route, const int32_t* cu_seqlens,
                             int batch, int max_seqlen, int hkv, int block_m,
                             int block_n, int group, uint64_t* mask,
                             int32_t* status, cudaStream_t stream);

// Routing-template layouts (same values as TILEMIX_LAYOUT_*).
constexpr int kLayoutAllFp16 = 0, kLayoutAllInt8 = 1, kLayoutBand = 2,
              kLayoutGlobal = 3, kLayoutRowRandom = 4, kLayoutAligned = 5,
              kLayoutBigBird = 6, kLayoutSpTrans = 7;

cudaError_t launch_route_template(int layout, int permille, uint64_t seed,
                                  const int32_t* cu_seqlens, int batch,
                                  int max_seqlen, int hkv, int block_m,
                                  int block_n, int group, uint8_t* route,
                                  int32_t* status, cudaStream_t stream);

size_t route_adaptive_workspace(int batch, int max_seqlen, int hkv, int d,
                                int block_m);
cudaError_t launch_route_adaptive(const void* q, const void* k,
                                  const int32_t* cu_seqlens, int batch,
                                  int max_seqlen, int total_tokens, int hq,
                                  int hkv, int d, const int32_t* head_map,
                                  int block_m, int block_n, int group,
                                  int permille, void* workspace, uint8_t* route,
                                  uint64_t* mask, int32_t* status,
                                  cudaStream_t stream);

// Device address (in the current context) of the file-scope scratch array
// that tilemix_route_adaptive_noalloc uses; looked up on every call.
cudaError_t route_adaptive_static_scratch(void** ptr);

// Everything the fused attention kernel reads.  Passed by value as a
// __grid_constant__ parameter; the tensor maps must stay 64-byte aligned.
struct AttnParams {
  CUtensorMap tm_q;   // fp16 Q  [T, hq, d], box {64, 128, 1}, 128B swizzle
  CUtensorMap tm_q8;  // int8 Q8 [T, hq, d], box {d, 128, 1}
  CUtensorMap tm_k;   // fp16 K  [T, hkv, d], box {64, 128, 1}
  CUtensorMap tm_k8;  // int8 K8 [T, hkv, d], box {d, 128, 1}
  CUtensorMap tm_v;   // fp16 V  [T, hkv, d], box {64, 128, 1}
  CUtensorMap tm_v8;  // int8 V8 [T, hkv, d], box {d, 128, 1}, no swizzle
  CUtensorMap tm_o;   // fp16 O  [T, hq, d], box {64, 128, 1}, 128B swizzle
  const uint16_t* k;  // fp16 K bits [T, hkv, d] (on-chip quantisation reads it)
  const int32_t* cu_seqlens;
  const int32_t* head_map;
  const uint64_t* mask;
  const float* q_scale;
  const float* k_scale;
  const float* v_scale;  // INT8 KV cache: [hkv, batch, nbk]
  uint16_t* out;     // fp16 bits [T, hq, d]
  float* lse;
  int32_t* qk_dump;
  int32_t* status;
  int batch, max_seqlen, total_tokens;
  int hq, hkv, heads_per_kv;
  int route_bm;      // 64 or 128: query rows per routing word
  int route_bn;      // 64 or 128: keys per routing (score) tile
  int tm_route;      // ceil(max_seqlen / route_bm)
  int tn_max;        // ceil(max_seqlen / route_bn)
  int group;         // g: routing tiles per bit
  int tiles_per_bit; // 64-key blocks per routing bit = g * route_bn / 64
  int quant_block_q, quant_block_k, nbq, nbk;
  int fp16_only;
  int test_expire_wait;
  int pv_f16_acc;  // study: O accumulated in fp16 (low half of each column)  // withhold the first V tile (timeout-path test)
  float scale_log2;  // softmax scale * log2(e)
};

struct AttnLaunchShape {
  int head_dim;
  bool dual;  // routing rows of 64 inside 128-row compute tiles
  // 0: Q8/K8 + scales given; 1: INT8 KV cache (k8, v8 + block scales);
  // 2: Q8/K8 + scales made on chip for INT8-routed tiles
  int mode;
};

cudaError_t launch_attn_prefill(const AttnParams& p, const AttnLaunchShape& s,
                                cudaStream_t stream);

// Dynamic shared memory and TMEM columns a shape needs (host query).
int attn_smem_bytes(const AttnLaunchShape& s);

}  // namespace tilemix
