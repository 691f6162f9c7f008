// Split-softmax GQA decode attention over a per-sequence K/V cache.
//
// Definition: turbospark-runtime 0.3.0, src/qwen3_asr_metal.rs, `step`
// (encode_attention_decode over rows [kv_start = 0, position] with the
// split-softmax AttentionScratch, scale 1/sqrt(head_dim)); makima
// src/tts/qwen3/model.rs, Qwen3Attention::forward and repeat_kv (query head
// h reads KV head h / (H/Hkv)).
//
// Grid (splits, Hkv, B). The CTA for split s of KV head kv scores the rows
// [s*CH, (s+1)*CH) of that head for all H/Hkv query heads that share it,
// keeping a running (max, sum, weighted V) per head (online softmax). Its
// partial goes to the workspace; the last CTA of a (b, kv) pair to finish
// (counted with an atomic ticket) merges all splits in split order, so the
// result does not depend on which CTA finishes last.
//
// Cache layout [B][Hkv][cap][D]: the rows of one head are contiguous, so a
// split reads one contiguous CH*D*2-byte run of K and one of V.
#include <mutex>

#include "attention_body.cuh"

namespace qg {

constexpr int kAttnWarps = 4;

struct AttnPlan {
  int ch;      // rows per split
  int nsplit;  // splits per (b, kv)
};

static AttnPlan attn_plan(int B, int Hkv, int cap) {
  // About four CTAs per SM across B * Hkv * splits, splits of 32 to 256 rows
  // (a warp then walks at most 64 rows, 8 of them in flight at a time); the
  // last CTA of each (sequence, kv head) merges the splits.
  const long long want = 4LL * 148;
  long long ch = ((long long)cap * B * Hkv + want - 1) / want;
  ch = ((ch + 31) / 32) * 32;
  if (ch < 32) ch = 32;
  if (ch > 256) ch = 256;
  AttnPlan p;
  p.ch = (int)ch;
  p.nsplit = (int)((cap + ch - 1) / ch);
  return p;
}

static size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

size_t attention_ws_bytes(int B, int H, int Hkv, int D, int cap) {
  const AttnPlan p = attn_plan(B, Hkv, cap);
  const size_t o = (size_t)B * H * p.nsplit * D * sizeof(float);
  const size_t ml = (size_t)B * H * p.nsplit * 2 * sizeof(float);
  const size_t cnt = (size_t)B * Hkv * sizeof(unsigned int);
  return align256(o) + align256(ml) + align256(cnt);
}

template <int VPL>  // values of a head row per lane: D = 32 * VPL
__global__ void __launch_bounds__(kAttnWarps * 32)
attention_split_kernel(const float* __restrict__ q, const uint16_t* __restrict__ kc,
                       const uint16_t* __restrict__ vc, const int32_t* __restrict__ kv_len,
                       const int32_t* __restrict__ pos_for_len, void* __restrict__ out,
                       int out_bf16, int H, int Hkv, int cap, float scale, int ch, int nsplit,
                       float* __restrict__ ws_o, float* __restrict__ ws_ml,
                       unsigned int* __restrict__ ws_cnt, const AttnFuse fz) {
  attention_body<VPL, kAttnWarps, kMaxGroup>(
      q, kc, vc, kv_len, pos_for_len, out, out_bf16, H, Hkv, cap, scale, ch, nsplit, ws_o, ws_ml,
      ws_cnt, fz, blockIdx.x, blockIdx.y, blockIdx.z, [] {
        // the next kernel may be scheduled now: its own wait covers all of this one
        pdl_trigger();
        pdl_wait();
      });
}

static cudaError_t attention_launch_any(const float* q, const uint16_t* kc, const uint16_t* vc,
                                        const int32_t* kv_len, const int32_t* pos_for_len,
                                        void* out, bool out_bf16, int B, int H, int Hkv, int D,
                                        int cap, float scale, void* ws, cudaStream_t st, bool pdl,
                                        const AttnFuse& fz) {
  const AttnPlan p = attn_plan(B, Hkv, cap);
  uint8_t* w = reinterpret_cast<uint8_t*>(ws);
  float* ws_o = reinterpret_cast<float*>(w);
  w += align256((size_t)B * H * p.nsplit * D * sizeof(float));
  float* ws_ml = reinterpret_cast<float*>(w);
  w += align256((size_t)B * H * p.nsplit * 2 * sizeof(float));
  unsigned int* ws_cnt = reinterpret_cast<unsigned int*>(w);
  dim3 grid(p.nsplit, Hkv, B), block(kAttnWarps * 32);
#define QG_ATTN_CASE(V)                                                                        \
  case V:                                                                                      \
    return launch_pdl(attention_split_kernel<V>, grid, block, 0, st, pdl, q, kc, vc, kv_len,   \
                      pos_for_len, out, (int)out_bf16, H, Hkv, cap, scale, p.ch, p.nsplit,     \
                      ws_o, ws_ml, ws_cnt, fz);
  switch (D / 32) {
    QG_ATTN_CASE(1)
    QG_ATTN_CASE(2)
    QG_ATTN_CASE(3)
    QG_ATTN_CASE(4)
    QG_ATTN_CASE(5)
    QG_ATTN_CASE(6)
    QG_ATTN_CASE(7)
    QG_ATTN_CASE(8)
    default:
      return cudaErrorInvalidValue;
  }
#undef QG_ATTN_CASE
}

cudaError_t attention_launch(const float* q, const uint16_t* kc, const uint16_t* vc,
                             const int32_t* kv_len, const int32_t* pos_for_len, void* out,
                             bool out_bf16, int B, int H, int Hkv, int D, int cap, float scale,
                             void* ws, cudaStream_t st, bool pdl) {
  AttnFuse fz = {};
  return attention_launch_any(q, kc, vc, kv_len, pos_for_len, out, out_bf16, B, H, Hkv, D, cap,
                              scale, ws, st, pdl, fz);
}

cudaError_t attention_launch_step(const float* q, const float* k, const float* v,
                                  const uint16_t* q_norm, const uint16_t* k_norm,
                                  const int32_t* tokens, int vocab, float eps, const float2* rope,
                                  uint16_t* kc, uint16_t* vc, const int32_t* positions, void* out,
                                  int B, int H, int Hkv, int D, int cap, float scale, void* ws,
                                  cudaStream_t st, bool pdl) {
  AttnFuse fz = {1, k, v, q_norm, k_norm, tokens, vocab, eps, rope};
  return attention_launch_any(q, kc, vc, nullptr, positions, out, true, B, H, Hkv, D, cap, scale,
                              ws, st, pdl, fz);
}

void attention_plan(int B, int Hkv, int cap, int* ch, int* nsplit) {
  const AttnPlan p = attn_plan(B, Hkv, cap);
  *ch = p.ch;
  *nsplit = p.nsplit;
}

void attention_ws_split(void* ws, int B, int H, int Hkv, int D, int cap, float** ws_o,
                        float** ws_ml, unsigned int** ws_cnt) {
  const AttnPlan p = attn_plan(B, Hkv, cap);
  uint8_t* w = reinterpret_cast<uint8_t*>(ws);
  *ws_o = reinterpret_cast<float*>(w);
  w += align256((size_t)B * H * p.nsplit * D * sizeof(float));
  *ws_ml = reinterpret_cast<float*>(w);
  w += align256((size_t)B * H * p.nsplit * 2 * sizeof(float));
  *ws_cnt = reinterpret_cast<unsigned int*>(w);
}

// Offset of the ticket counters inside an attention workspace.
size_t attention_ws_counter_offset(int B, int H, int Hkv, int D, int cap) {
  const AttnPlan p = attn_plan(B, Hkv, cap);
  return align256((size_t)B * H * p.nsplit * D * sizeof(float)) +
         align256((size_t)B * H * p.nsplit * 2 * sizeof(float));
}

}  // namespace qg

using namespace qg;

static qg_status validate_attention(const float* q, const uint16_t* kc, const uint16_t* vc,
                                    const int32_t* kv_len, void* out, qg_dtype od, int B, int H,
                                    int Hkv, int D, int cap) {
  QG_REQUIRE(B >= 0 && H >= 1 && Hkv >= 1, QG_ERR_UNSUPPORTED_SHAPE,
             "qg_decode_attention: B=%d H=%d Hkv=%d", B, H, Hkv);
  QG_REQUIRE(H % Hkv == 0 && H / Hkv <= kMaxGroup, QG_ERR_UNSUPPORTED_SHAPE,
             "qg_decode_attention: H=%d must be a multiple of Hkv=%d with H/Hkv <= 8", H, Hkv);
  QG_REQUIRE(D >= 32 && D <= 256 && D % 32 == 0, QG_ERR_UNSUPPORTED_SHAPE,
             "qg_decode_attention: D=%d must be a multiple of 32 in [32, 256]", D);
  QG_REQUIRE(cap >= 1, QG_ERR_UNSUPPORTED_SHAPE, "qg_decode_attention: cap=%d must be >= 1", cap);
  QG_REQUIRE(od == QG_F32 || od == QG_BF16, QG_ERR_INVALID_ARGUMENT,
             "qg_decode_attention: out_dtype=%d is not QG_F32 or QG_BF16", (int)od);
  QG_REQUIRE((long long)B * Hkv * cap * D < (1LL << 40), QG_ERR_UNSUPPORTED_SHAPE,
             "qg_decode_attention: cache too large");
  if (B == 0) return QG_OK;
  QG_REQUIRE(q && kc && vc && kv_len && out, QG_ERR_INVALID_ARGUMENT,
             "qg_decode_attention: null q, k_cache, v_cache, kv_len or out");
  QG_REQUIRE(aligned(q, 16) && aligned(kc, 16) && aligned(vc, 16) && aligned(out, 16),
             QG_ERR_MISALIGNED, "qg_decode_attention: q, k_cache, v_cache or out not 16-byte aligned");
  QG_REQUIRE(aligned(kv_len, 4), QG_ERR_MISALIGNED, "qg_decode_attention: kv_len misaligned");
  return QG_OK;
}

extern "C" size_t qg_decode_attention_workspace_size(int B, int H, int Hkv, int D, int cap) {
  if (B <= 0 || H <= 0 || Hkv <= 0 || D <= 0 || cap <= 0) return 0;
  return attention_ws_bytes(B, H, Hkv, D, cap);
}

extern "C" qg_status qg_decode_attention(const float* q, const uint16_t* k_cache,
                                         const uint16_t* v_cache, const int32_t* kv_len, void* out,
                                         qg_dtype out_dtype, int B, int H, int Hkv, int D, int cap,
                                         float scale, void* ws, size_t ws_bytes, void* stream) {
  clear_error();
  qg_status st = validate_attention(q, k_cache, v_cache, kv_len, out, out_dtype, B, H, Hkv, D, cap);
  if (st != QG_OK || B == 0) return st;
  const size_t need = attention_ws_bytes(B, H, Hkv, D, cap);
  QG_REQUIRE(ws && ws_bytes >= need, QG_ERR_WORKSPACE_TOO_SMALL,
             "qg_decode_attention: workspace of %zu bytes given, %zu needed", ws_bytes, need);
  QG_REQUIRE(aligned(ws, 256), QG_ERR_MISALIGNED, "qg_decode_attention: ws not 256-byte aligned");
  cudaStream_t s = (cudaStream_t)stream;
  const size_t off = attention_ws_counter_offset(B, H, Hkv, D, cap);
  cudaMemsetAsync(reinterpret_cast<uint8_t*>(ws) + off, 0, (size_t)B * Hkv * sizeof(unsigned int), s);
  attention_launch(q, k_cache, v_cache, kv_len, nullptr, out, out_dtype == QG_BF16, B, H, Hkv, D,
                   cap, scale, ws, s, false);
  return check_launch("qg_decode_attention");
}

// --------------------------------------------------------------------------
// qg_decode_attention_static_scratch: the same attention with its scratch in
// a fixed device array of this library instead of a caller workspace.
//
// Some callers cannot hand the library device memory at the point of the
// call: a plain C host that holds only the cache and activation buffers
// and no device allocator, or a decode loop that must not call cudaMalloc /
// cudaFree between steps (cudaFree synchronises the device, cudaMalloc may).
// This entry point allocates nothing: its split partials and ticket
// counters live in g_attn_scratch below, a file-scope device array of
// kAttnStaticScratchBytes, whose address the host looks up once per device.
// --------------------------------------------------------------------------

namespace qg {

constexpr size_t kAttnStaticScratchBytes = 4u << 20;  // 4 MiB per device
static __device__ __align__(256) uint8_t g_attn_scratch[kAttnStaticScratchBytes];

constexpr int kMaxDevices = 64;

// Device address of g_attn_scratch on the current device, looked up once per
// device (with that device current) and cached.
static cudaError_t attn_scratch_address(void** out) {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_attn_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
  }
  *out = addr[dev];
  return cudaSuccess;
}

}  // namespace qg

extern "C" size_t qg_decode_attention_static_scratch_capacity(void) {
  return kAttnStaticScratchBytes;
}

extern "C" qg_status qg_decode_attention_static_scratch(const float* q, const uint16_t* k_cache,
                                                        const uint16_t* v_cache,
                                                        const int32_t* kv_len, void* out,
                                                        qg_dtype out_dtype, int B, int H, int Hkv,
                                                        int D, int cap, float scale,
                                                        void* stream) {
  clear_error();
  qg_status st = validate_attention(q, k_cache, v_cache, kv_len, out, out_dtype, B, H, Hkv, D, cap);
  if (st != QG_OK || B == 0) return st;
  const size_t need = attention_ws_bytes(B, H, Hkv, D, cap);
  QG_REQUIRE(need <= kAttnStaticScratchBytes, QG_ERR_WORKSPACE_TOO_SMALL,
             "qg_decode_attention_static_scratch: this shape needs %zu bytes of scratch, more "
             "than the fixed %zu; use qg_decode_attention with a caller workspace",
             need, kAttnStaticScratchBytes);
  void* ws = nullptr;
  cudaError_t e = attn_scratch_address(&ws);
  if (e != cudaSuccess) {
    set_error("qg_decode_attention_static_scratch: scratch address lookup failed: %s",
              cudaGetErrorString(e));
    return QG_ERR_CUDA;
  }
  cudaStream_t s = (cudaStream_t)stream;
  // the ticket counters must start at zero (the kernel also leaves them at
  // zero; a cleared start does not depend on how the last call ended)
  const size_t off = attention_ws_counter_offset(B, H, Hkv, D, cap);
  e = cudaMemsetAsync(reinterpret_cast<uint8_t*>(ws) + off, 0, (size_t)B * Hkv * sizeof(unsigned int), s);
  if (e != cudaSuccess) {
    set_error("qg_decode_attention_static_scratch: %s", cudaGetErrorString(e));
    return QG_ERR_CUDA;
  }
  attention_launch(q, k_cache, v_cache, kv_len, nullptr, out, out_dtype == QG_BF16, B, H, Hkv, D,
                   cap, scale, ws, s, false);
  return check_launch("qg_decode_attention_static_scratch");
}
