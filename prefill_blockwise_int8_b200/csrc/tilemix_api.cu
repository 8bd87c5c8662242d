// C ABI of the library (declared in include/tilemix.h): argument checks,
// TMA tensor-map construction and kernel dispatch.  Host code only; it never
// allocates, synchronises or copies.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "internal.h"
#include "tilemix.h"

namespace {

thread_local std::string g_last_error;

tilemix_status fail(tilemix_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

tilemix_status ok() {
  g_last_error.clear();
  return TILEMIX_OK;
}

bool aligned(const void* p, size_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

tilemix_status check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess)
    return fail(TILEMIX_ERR_NO_DEVICE, "no CUDA device");
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0)
    return fail(TILEMIX_ERR_NO_DEVICE,
                "device %d is sm_%d%d; this library is built for sm_100a", dev,
                major, minor);
  return TILEMIX_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault,
                                &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3-D map over a token-major [T, H, d] tensor: dims {d, T, H}; a box of
// {box_x elements, box_rows tokens, 1 head}.
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt,
              int elem_bytes, int d, int tokens, int heads, int box_x,
              int box_rows, CUtensorMapSwizzle sw) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d),
                        static_cast<cuuint64_t>(tokens),
                        static_cast<cuuint64_t>(heads)};
  cuuint64_t strides[2] = {
      static_cast<cuuint64_t>(heads) * d * elem_bytes,
      static_cast<cuuint64_t>(d) * elem_bytes};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box_x),
                       static_cast<cuuint32_t>(box_rows), 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

extern "C" {

const char* tilemix_status_string(tilemix_status s) {
  switch (s) {
    case TILEMIX_OK: return "ok";
    case TILEMIX_ERR_INVALID_ARG: return "invalid argument";
    case TILEMIX_ERR_UNSUPPORTED: return "unsupported configuration";
    case TILEMIX_ERR_CUDA: return "CUDA error";
    case TILEMIX_ERR_TIMEOUT: return "device pipeline wait timed out";
    case TILEMIX_ERR_BAD_SEQLENS: return "invalid cu_seqlens or head_map";
    case TILEMIX_ERR_NO_DEVICE: return "no sm_100 device";
  }
  return "unknown status";
}

const char* tilemix_last_error(void) { return g_last_error.c_str(); }

uint32_t tilemix_version(void) { return (1u << 16) | 0u; }

tilemix_status tilemix_quantize_blockwise(const void* x,
                                          const int32_t* cu_seqlens, int batch,
                                          int max_seqlen, int total_tokens,
                                          int heads, int head_dim, int block,
                                          int8_t* x8, float* scale,
                                          int32_t* status,
                                          tilemix_stream_t stream) {
  if (!x || !cu_seqlens || !x8 || !scale)
    return fail(TILEMIX_ERR_INVALID_ARG, "quantize: null pointer");
  if (!aligned(x, 16) || !aligned(x8, 16) || !aligned(scale, 4) ||
      !aligned(cu_seqlens, 4) || (status && !aligned(status, 4)))
    return fail(TILEMIX_ERR_INVALID_ARG, "quantize: misaligned pointer");
  if (batch < 0 || max_seqlen < 0 || total_tokens < 0 || heads <= 0)
    return fail(TILEMIX_ERR_INVALID_ARG, "quantize: negative size");
  if (head_dim <= 0 || head_dim % 8 != 0 || head_dim > 256)
    return fail(TILEMIX_ERR_INVALID_ARG,
                "quantize: head_dim %d must be a multiple of 8 in [8, 256]",
                head_dim);
  if (block <= 0 || block > 256 || block * head_dim > 32768)
    return fail(TILEMIX_ERR_INVALID_ARG,
                "quantize: block %d out of range (block*head_dim <= 32768)",
                block);
  if (batch == 0 || max_seqlen == 0) return ok();
  if ((max_seqlen + block - 1) / block > 2147483647)
    return fail(TILEMIX_ERR_INVALID_ARG, "quantize: too many blocks");
  if (heads > 65535 || batch > 65535)
    return fail(TILEMIX_ERR_UNSUPPORTED, "quantize: heads/batch > 65535");
  tilemix_status d = check_device();
  if (d != TILEMIX_OK) return d;
  cudaError_t e = tilemix::launch_quantize_blockwise(
      x, cu_seqlens, batch, max_seqlen, total_tokens, heads, head_dim, block,
      x8, scale, status, stream);
  if (e != cudaSuccess)
    return fail(TILEMIX_ERR_CUDA, "quantize launch: %s", cudaGetErrorString(e));
  return ok();
}

tilemix_status tilemix_quantize_blockwise_qk(
    const void* q, const void* k, const int32_t* cu_seqlens, int batch,
    int max_seqlen, int total_tokens, int hq, int hkv, int head_dim,
    int block_q, int block_k, int8_t* q8, float* q_scale, int8_t* k8,
    float* k_scale, int32_t* status, tilemix_stream_t stream) {
  if (!q || !k || !cu_seqlens || !q8 || !q_scale || !k8 || !k_scale)
    return fail(TILEMIX_ERR_INVALID_ARG, "quantize_qk: null pointer");
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(q8, 16) ||
      !aligned(k8, 16) || !aligned(q_scale, 4) || !aligned(k_scale, 4) ||
      !aligned(cu_seqlens, 4) || (status && !aligned(status, 4)))
    return fail(TILEMIX_ERR_INVALID_ARG, "quantize_qk: misaligned pointer");
  if (batch < 0 || max_seqlen < 0 || total_tokens < 0 || hq <= 0 || hkv <= 0)
    return fail(TILEMIX_ERR_INVALID_ARG, "quantize_qk: negative size");
  if (head_dim <= 0 || head_dim % 8 != 0 || head_dim > 256)
    return fail(TILEMIX_ERR_INVALID_ARG,
                "quantize_qk: head_dim %d must be a multiple of 8 in [8, 256]",
                head_dim);
  for (int blk : {block_q, block_k})
    if (blk <= 0 || blk > 256 || blk * head_dim > 32768)
      return fail(TILEMIX_ERR_INVALID_ARG,
                  "quantize_qk: block %d out of range (block*head_dim <= 32768)",
                  blk);
  if (batch == 0 || max_seqlen == 0) return ok();
  if (static_cast<long long>(hq) + hkv > 65535 || batch > 65535)
    return fail(TILEMIX_ERR_UNSUPPORTED,
                "quantize_qk: hq + hkv or batch > 65535");
  tilemix_status d = check_device();
  if (d != TILEMIX_OK) return d;
  cudaError_t e = tilemix::launch_quantize_blockwise_qk(
      q, k, cu_seqlens, batch, max_seqlen, total_tokens, hq, hkv, head_dim,
      block_q, block_k, q8, q_scale, k8, k_scale, status, stream);
  if (e != cudaSuccess)
    return fail(TILEMIX_ERR_CUDA, "quantize_qk launch: %s",
                cudaGetErrorString(e));
  return ok();
}

tilemix_status tilemix_pack_mask(const uint8_t* route,
                                 const int32_t* cu_seqlens, int batch,
                                 int max_seqlen, int hkv, int block_m,
                                 int block_n, int group, uint64_t* mask,
                                 int32_t* status, tilemix_stream_t stream) {
  if (!route || !cu_seqlens || !mask)
    return fail(TILEMIX_ERR_INVALID_ARG, "pack_mask: null pointer");
  if (!aligned(route, 16) || !aligned(mask, 8) || !aligned(cu_seqlens, 4) ||
      (status && !aligned(status, 4)))
    return fail(TILEMIX_ERR_INVALID_ARG, "pack_mask: misaligned pointer");
  if (batch < 0 || max_seqlen < 0 || hkv <= 0 || block_m <= 0 ||
      block_n <= 0 || group <= 0)
    return fail(TILEMIX_ERR_INVALID_ARG, "pack_mask: bad size");
  if (batch == 0 || max_seqlen == 0) return ok();
  const long long tn = (static_cast<long long>(max_seqlen) + block_n - 1) / block_n;
  if ((tn + group - 1) / group > 64)
    return fail(TILEMIX_ERR_INVALID_ARG,
                "pack_mask: ceil(%lld key tiles / g=%d) > 64 routing bits", tn,
                group);
  tilemix_status d = check_device();
  if (d != TILEMIX_OK) return d;
  cudaError_t e =
      tilemix::launch_pack_mask(route, cu_seqlens, batch, max_seqlen, hkv,
                                block_m, block_n, group, mask, status, stream);
  if (e != cudaSuccess)
    return fail(TILEMIX_ERR_CUDA, "pack_mask launch: %s", cudaGetErrorString(e));
  return ok();
}

tilemix_status tilemix_route_template(int layout, int int8_permille,
                                      uint64_t seed, const int32_t* cu_seqlens,
                                      int batch, int max_seqlen, int hkv,
                                      int block_m, int block_n, int group,
                                      uint8_t* route, int32_t* status,
                                      tilemix_stream_t stream) {
  if (!route || !cu_seqlens)
    return fail(TILEMIX_ERR_INVALID_ARG, "route_template: null pointer");
  if (!aligned(route, 16) || !aligned(cu_seqlens, 4) ||
      (status && !aligned(status, 4)))
    return fail(TILEMIX_ERR_INVALID_ARG, "route_template: misaligned pointer");
  if (layout < TILEMIX_LAYOUT_ALL_FP16 || layout > TILEMIX_LAYOUT_SPTRANS)
    return fail(TILEMIX_ERR_INVALID_ARG, "route_template: bad layout %d",
                layout);
  if (int8_permille < 0 || int8_permille > 1000)
    return fail(TILEMIX_ERR_INVALID_ARG,
                "route_template: int8_permille %d not in [0, 1000]",
                int8_permille);
  if (batch < 0 || max_seqlen < 0 || hkv <= 0 || block_m <= 0 ||
      block_n <= 0 || group <= 0)
    return fail(TILEMIX_ERR_INVALID_ARG, "route_template: bad size");
  if (batch == 0 || max_seqlen == 0) return ok();
  const long long tn = (static_cast<long long>(max_seqlen) + block_n - 1) / block_n;
  if ((tn + group - 1) / group > 64)
    return fail(TILEMIX_ERR_INVALID_ARG,
                "route_template: ceil(%lld key tiles / g=%d) > 64 routing bits",
                tn, group);
  tilemix_status d = check_device();
  if (d != TILEMIX_OK) return d;
  cudaError_t e = tilemix::launch_route_template(
      layout, int8_permille, seed, cu_seqlens, batch, max_seqlen, hkv, block_m,
      block_n, group, route, status, stream);
  if (e != cudaSuccess)
    return fail(TILEMIX_ERR_CUDA, "route_template launch: %s",
                cudaGetErrorString(e));
  return ok();
}

size_t tilemix_route_adaptive_workspace_bytes(int batch, int max_seqlen,
                                              int hkv, int head_dim,
                                              int block_m) {
  if (batch < 0 || max_seqlen < 0 || hkv <= 0 || head_dim <= 0 || block_m <= 0)
    return 0;
  return tilemix::route_adaptive_workspace(batch, max_seqlen, hkv, head_dim,
                                           block_m);
}

namespace {

// Host checks shared by both adaptive-routing entry points.  On TILEMIX_OK,
// *need is the scratch the two passes use (0 when there is nothing to do).
tilemix_status route_adaptive_check(
    const char* where, const void* q, const void* k, const int32_t* cu_seqlens,
    int batch, int max_seqlen, int total_tokens, int hq, int hkv, int head_dim,
    const int32_t* head_map, int block_m, int block_n, int group,
    int int8_permille, const uint8_t* route, const uint64_t* mask,
    const int32_t* status, size_t* need) {
  *need = 0;
  if (!q || !k || !cu_seqlens || (!route && !mask))
    return fail(TILEMIX_ERR_INVALID_ARG, "%s: null pointer", where);
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(route, 16) ||
      !aligned(mask, 8) || !aligned(cu_seqlens, 4) ||
      (head_map && !aligned(head_map, 4)) || (status && !aligned(status, 4)))
    return fail(TILEMIX_ERR_INVALID_ARG, "%s: misaligned pointer", where);
  if (int8_permille < 0 || int8_permille > 1000)
    return fail(TILEMIX_ERR_INVALID_ARG, "%s: int8_permille %d not in [0, 1000]",
                where, int8_permille);
  if (batch < 0 || max_seqlen < 0 || total_tokens < 0 || hq <= 0 || hkv <= 0 ||
      block_m <= 0 || block_n <= 0 || group <= 0)
    return fail(TILEMIX_ERR_INVALID_ARG, "%s: bad size", where);
  if (head_dim < 8 || head_dim > 256 || head_dim % 8 != 0)
    return fail(TILEMIX_ERR_UNSUPPORTED,
                "%s: head_dim %d not a multiple of 8 in [8, 256]", where,
                head_dim);
  if (!head_map && hq % hkv != 0)
    return fail(TILEMIX_ERR_INVALID_ARG,
                "%s: hq %d not a multiple of hkv %d and no head_map", where, hq,
                hkv);
  if (hkv > 65535 || batch > 65535)
    return fail(TILEMIX_ERR_UNSUPPORTED, "%s: hkv or batch > 65535", where);
  if (batch == 0 || max_seqlen == 0) return ok();
  const long long tn = (static_cast<long long>(max_seqlen) + block_n - 1) / block_n;
  if ((tn + group - 1) / group > 64)
    return fail(TILEMIX_ERR_INVALID_ARG,
                "%s: ceil(%lld key tiles / g=%d) > 64 routing bits", where, tn,
                group);
  // |fp16 * 2^24| < 2^40, so a tile's query sums stay below 2^40 * rows and
  // a group's key sums below 2^40 * keys; the device's 24-bit limb products
  // and the int128 statistic stay exact within these bounds.
  const long long rows = static_cast<long long>(block_m) * (head_map ? hq : hq / hkv);
  const long long keys = static_cast<long long>(group) * block_n;
  if (rows >= (1ll << 15) || keys >= (1ll << 15) ||
      rows * head_dim >= (1ll << 22) || keys * head_dim >= (1ll << 22) ||
      rows * keys * head_dim >= (1ll << 47))
    return fail(TILEMIX_ERR_UNSUPPORTED,
                "%s: tile sizes too large for exact statistics", where);
  const long long tm = (static_cast<long long>(max_seqlen) + block_m - 1) / block_m;
  if (static_cast<long long>(batch) * hkv * tm > 0x7fffffffll)
    return fail(TILEMIX_ERR_UNSUPPORTED, "%s: too many routing rows", where);
  *need = tilemix::route_adaptive_workspace(batch, max_seqlen, hkv, head_dim,
                                            block_m);
  return ok();
}

}  // namespace

tilemix_status tilemix_route_adaptive(
    const void* q, const void* k, const int32_t* cu_seqlens, int batch,
    int max_seqlen, int total_tokens, int hq, int hkv, int head_dim,
    const int32_t* head_map, int block_m, int block_n, int group,
    int int8_permille, void* workspace, size_t workspace_bytes,
    uint8_t* route, uint64_t* mask, int32_t* status, tilemix_stream_t stream) {
  size_t need = 0;
  tilemix_status st = route_adaptive_check(
      "route_adaptive", q, k, cu_seqlens, batch, max_seqlen, total_tokens, hq,
      hkv, head_dim, head_map, block_m, block_n, group, int8_permille, route,
      mask, status, &need);
  if (st != TILEMIX_OK || need == 0) return st;
  if (!workspace || !aligned(workspace, 16) || workspace_bytes < need)
    return fail(TILEMIX_ERR_INVALID_ARG,
                "route_adaptive: workspace of %zu bytes (16-byte aligned) "
                "needed, %zu given",
                need, workspace ? workspace_bytes : static_cast<size_t>(0));
  tilemix_status d = check_device();
  if (d != TILEMIX_OK) return d;
  cudaError_t e = tilemix::launch_route_adaptive(
      q, k, cu_seqlens, batch, max_seqlen, total_tokens, hq, hkv, head_dim,
      head_map, block_m, block_n, group, int8_permille, workspace, route,
      mask, status, stream);
  if (e != cudaSuccess)
    return fail(TILEMIX_ERR_CUDA, "route_adaptive launch: %s",
                cudaGetErrorString(e));
  return ok();
}

tilemix_status tilemix_route_adaptive_noalloc(
    const void* q, const void* k, const int32_t* cu_seqlens, int batch,
    int max_seqlen, int total_tokens, int hq, int hkv, int head_dim,
    const int32_t* head_map, int block_m, int block_n, int group,
    int int8_permille, uint8_t* route, uint64_t* mask, int32_t* status,
    tilemix_stream_t stream) {
  size_t need = 0;
  tilemix_status st = route_adaptive_check(
      "route_adaptive_noalloc", q, k, cu_seqlens, batch, max_seqlen,
      total_tokens, hq, hkv, head_dim, head_map, block_m, block_n, group,
      int8_permille, route, mask, status, &need);
  if (st != TILEMIX_OK || need == 0) return st;
  if (need > TILEMIX_ROUTE_ADAPTIVE_STATIC_BYTES)
    return fail(TILEMIX_ERR_INVALID_ARG,
                "route_adaptive_noalloc: %zu bytes of scratch needed, the "
                "static scratch holds %zu",
                need, static_cast<size_t>(TILEMIX_ROUTE_ADAPTIVE_STATIC_BYTES));
  tilemix_status d = check_device();
  if (d != TILEMIX_OK) return d;
  void* scratch = nullptr;
  cudaError_t e = tilemix::route_adaptive_static_scratch(&scratch);
  if (e != cudaSuccess)
    return fail(TILEMIX_ERR_CUDA, "route_adaptive_noalloc scratch: %s",
                cudaGetErrorString(e));
  e = tilemix::launch_route_adaptive(
      q, k, cu_seqlens, batch, max_seqlen, total_tokens, hq, hkv, head_dim,
      head_map, block_m, block_n, group, int8_permille, scratch, route, mask,
      status, stream);
  if (e != cudaSuccess)
    return fail(TILEMIX_ERR_CUDA, "route_adaptive_noalloc launch: %s",
                cudaGetErrorString(e));
  return ok();
}

tilemix_status tilemix_attn_prefill(const tilemix_attn_params* a,
                                    tilemix_stream_t stream) {
  if (!a) return fail(TILEMIX_ERR_INVALID_ARG, "attn: params is NULL");
  if (a->struct_size != sizeof(tilemix_attn_params))
    return fail(TILEMIX_ERR_INVALID_ARG,
                "attn: struct_size %u != sizeof(tilemix_attn_params) %zu",
                a->struct_size, sizeof(tilemix_attn_params));
  if (a->causal != 1)
    return fail(TILEMIX_ERR_UNSUPPORTED, "attn: only causal attention is built");
  const bool fp16_only = (a->flags & TILEMIX_FLAG_FP16_ONLY) != 0;
  // With every tile FP16 there is nothing to quantise on chip.
  const bool on_chip = !fp16_only && (a->flags & TILEMIX_FLAG_QUANT_ON_CHIP) != 0;
  if (a->flags & ~(TILEMIX_FLAG_FP16_ONLY | TILEMIX_FLAG_QUANT_ON_CHIP |
                   TILEMIX_FLAG_TEST_EXPIRE_WAIT | TILEMIX_FLAG_PV_F16_ACC))
    return fail(TILEMIX_ERR_INVALID_ARG, "attn: unknown flag bits 0x%x",
                a->flags);
  if (a->kv_format != TILEMIX_KV_FP16 && a->kv_format != TILEMIX_KV_INT8)
    return fail(TILEMIX_ERR_INVALID_ARG, "attn: bad kv_format %d", a->kv_format);
  const bool kv8 = a->kv_format == TILEMIX_KV_INT8;
  if (a->head_dim != 64 && a->head_dim != 128)
    return fail(TILEMIX_ERR_UNSUPPORTED, "attn: head_dim %d not in {64, 128}",
                a->head_dim);
  if (a->block_n != 64 && a->block_n != 128)
    return fail(TILEMIX_ERR_UNSUPPORTED, "attn: block_n %d not in {64, 128}",
                a->block_n);
  if (a->block_m != 64 && a->block_m != 128)
    return fail(TILEMIX_ERR_UNSUPPORTED, "attn: block_m %d not in {64, 128}",
                a->block_m);
  if (a->block_m == 64 && a->block_n != 64)
    return fail(TILEMIX_ERR_UNSUPPORTED, "attn: block_m 64 needs block_n 64");
  if (a->batch < 0 || a->max_seqlen < 0 || a->total_tokens < 0 ||
      a->hq <= 0 || a->hkv <= 0 || a->group <= 0)
    return fail(TILEMIX_ERR_INVALID_ARG, "attn: bad size");
  if (!a->head_map && a->hq % a->hkv != 0)
    return fail(TILEMIX_ERR_INVALID_ARG,
                "attn: hq %d not a multiple of hkv %d and no head_map", a->hq,
                a->hkv);
  // grid (hq, query-tile groups, batch): a CTA holds 256 query rows, or 128
  // with 64-row routing words (counted in 64 bits: max_seqlen may be near
  // INT_MAX)
  const long long rows_per_cta = a->block_m == 64 ? 128 : 256;
  const long long cta_rows =
      (static_cast<long long>(a->max_seqlen) + rows_per_cta - 1) / rows_per_cta;
  if (a->hq > 65535 || a->batch > 65535 || cta_rows > 65535)
    return fail(TILEMIX_ERR_UNSUPPORTED,
                "attn: hq, batch or query-tile groups per sequence above 65535");
  const int qbq = a->quant_block_q > 0 ? a->quant_block_q : 128;
  const int qbk = a->quant_block_k > 0 ? a->quant_block_k : 128;
  if (qbk % a->block_n != 0)
    return fail(TILEMIX_ERR_UNSUPPORTED,
                "attn: quant_block_k %d must be a multiple of block_n %d", qbk,
                a->block_n);
  const long long tn =
      (static_cast<long long>(a->max_seqlen) + a->block_n - 1) / a->block_n;
  if ((tn + a->group - 1) / a->group > 64)
    return fail(TILEMIX_ERR_INVALID_ARG,
                "attn: ceil(%lld key tiles / g=%d) > 64 routing bits", tn,
                a->group);
  if (!a->q || !a->out || !a->cu_seqlens)
    return fail(TILEMIX_ERR_INVALID_ARG, "attn: null q/out/cu_seqlens");
  if (!kv8 && (!a->k || !a->v))
    return fail(TILEMIX_ERR_INVALID_ARG, "attn: null k/v");
  if (kv8 && (!a->k8 || !a->k_scale || !a->v8 || !a->v_scale))
    return fail(TILEMIX_ERR_INVALID_ARG,
                "attn: the INT8 KV cache needs k8, k_scale, v8 and v_scale");
  if (on_chip && kv8)
    return fail(TILEMIX_ERR_UNSUPPORTED,
                "attn: on-chip quantisation needs the FP16 KV format");
  if (on_chip && (qbq != 128 || qbk != 128))
    return fail(TILEMIX_ERR_UNSUPPORTED,
                "attn: on-chip quantisation needs 128-token quantisation blocks");
  if (on_chip && !a->mask)
    return fail(TILEMIX_ERR_INVALID_ARG, "attn: mask is required");
  if (!fp16_only && !on_chip &&
      (!a->mask || !a->q8 || !a->q_scale || !a->k8 || !a->k_scale))
    return fail(TILEMIX_ERR_INVALID_ARG,
                "attn: mask, q8, q_scale, k8 and k_scale are required unless "
                "TILEMIX_FLAG_FP16_ONLY or TILEMIX_FLAG_QUANT_ON_CHIP is set");
  if (!aligned(a->q, 16) || (a->k && !aligned(a->k, 16)) ||
      (a->v && !aligned(a->v, 16)) || (a->v8 && !aligned(a->v8, 16)) ||
      (a->v_scale && !aligned(a->v_scale, 4)) ||
      !aligned(a->out, 16) || !aligned(a->cu_seqlens, 4) ||
      (a->q8 && !aligned(a->q8, 16)) || (a->k8 && !aligned(a->k8, 16)) ||
      (a->q_scale && !aligned(a->q_scale, 4)) ||
      (a->k_scale && !aligned(a->k_scale, 4)) ||
      (a->mask && !aligned(a->mask, 8)) || (a->lse && !aligned(a->lse, 4)) ||
      (a->qk_dump && !aligned(a->qk_dump, 4)) ||
      (a->head_map && !aligned(a->head_map, 4)) ||
      (a->status && !aligned(a->status, 4)))
    return fail(TILEMIX_ERR_INVALID_ARG, "attn: misaligned pointer");
  if (a->batch == 0 || a->max_seqlen == 0 || a->total_tokens == 0) return ok();
  tilemix_status dv = check_device();
  if (dv != TILEMIX_OK) return dv;
  if (!encode_fn())
    return fail(TILEMIX_ERR_CUDA, "attn: cuTensorMapEncodeTiled unavailable");

  const int d = a->head_dim;
  const int bn = a->block_n;
  const int T = a->total_tokens;
  tilemix::AttnParams p;
  memset(&p, 0, sizeof(p));
  const CUtensorMapSwizzle i8sw =
      d == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  // The kernel computes 128 x 128 score tiles (a 64-key routing tile is one
  // half of a compute tile).
  bool maps = make_map(&p.tm_q, a->q, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, d, T,
                       a->hq, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_map(&p.tm_o, a->out, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, d,
                       T, a->hq, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (maps && !kv8)
    maps = make_map(&p.tm_k, a->k, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, d, T,
                    a->hkv, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) &&
           make_map(&p.tm_v, a->v, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, d, T,
                    a->hkv, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (maps && !fp16_only && !on_chip)
    maps = make_map(&p.tm_q8, a->q8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, d, T,
                    a->hq, d, 128, i8sw);
  // The INT8 cache always feeds K8 (the INT8 path, or converted to fp16 on
  // chip for FP16 groups) and V8 (converted to fp16 on chip).
  if (maps && (kv8 || (!fp16_only && !on_chip)))
    maps = make_map(&p.tm_k8, a->k8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, d, T,
                    a->hkv, d, 128, i8sw);
  if (maps && kv8)
    maps = make_map(&p.tm_v8, a->v8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, d, T,
                    a->hkv, d, 128, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!maps) return fail(TILEMIX_ERR_CUDA, "attn: tensor map encoding failed");

  p.k = kv8 ? nullptr : static_cast<const uint16_t*>(a->k);
  p.cu_seqlens = a->cu_seqlens;
  p.head_map = a->head_map;
  p.mask = fp16_only ? nullptr : a->mask;
  p.q_scale = (fp16_only || on_chip) ? nullptr : a->q_scale;
  p.k_scale = ((fp16_only && !kv8) || on_chip) ? nullptr : a->k_scale;
  p.v_scale = kv8 ? a->v_scale : nullptr;
  p.out = static_cast<uint16_t*>(a->out);
  p.lse = a->lse;
  p.qk_dump = a->qk_dump;
  p.status = a->status;
  p.batch = a->batch;
  p.max_seqlen = a->max_seqlen;
  p.total_tokens = T;
  p.hq = a->hq;
  p.hkv = a->hkv;
  p.heads_per_kv = a->head_map ? 1 : a->hq / a->hkv;
  p.route_bm = a->block_m;
  p.route_bn = bn;
  p.tm_route = (a->max_seqlen + a->block_m - 1) / a->block_m;
  p.tn_max = (a->max_seqlen + bn - 1) / bn;
  p.group = a->group;
  p.tiles_per_bit = a->group * (bn / 64);
  p.quant_block_q = qbq;
  p.quant_block_k = qbk;
  p.nbq = (a->max_seqlen + qbq - 1) / qbq;
  p.nbk = (a->max_seqlen + qbk - 1) / qbk;
  p.fp16_only = fp16_only ? 1 : 0;
  p.test_expire_wait = (a->flags & TILEMIX_FLAG_TEST_EXPIRE_WAIT) ? 1 : 0;
  p.pv_f16_acc = (a->flags & TILEMIX_FLAG_PV_F16_ACC) ? 1 : 0;
  const float scale =
      a->softmax_scale > 0.0f ? a->softmax_scale : 1.0f / std::sqrt(float(d));
  p.scale_log2 = scale * 1.4426950408889634f;

  tilemix::AttnLaunchShape shape{d, a->block_m == 64, kv8 ? 1 : (on_chip ? 2 : 0)};
  const cudaError_t e = tilemix::launch_attn_prefill(p, shape, stream);
  if (e != cudaSuccess)
    return fail(TILEMIX_ERR_CUDA, "attn launch: %s", cudaGetErrorString(e));
  return ok();
}

}  // extern "C"
