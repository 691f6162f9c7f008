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
#include "qg_internal.cuh"

namespace qg {

constexpr int kAttnWarps = 4;
constexpr int kMaxGroup = 8;

struct AttnPlan {
  int ch;      // rows per split
  int nsplit;  // splits per (b, kv)
};

static AttnPlan attn_plan(int B, int Hkv, int cap) {
  // Aim for about two CTAs per SM across B * Hkv * splits.
  const long long want = 2LL * 148;
  long long ch = ((long long)cap * B * Hkv + want - 1) / want;
  ch = ((ch + 31) / 32) * 32;
  if (ch < 32) ch = 32;
  if (ch > 1024) ch = 1024;
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
                       unsigned int* __restrict__ ws_cnt) {
  constexpr int D = 32 * VPL;
  const int s = blockIdx.x, kv = blockIdx.y, b = blockIdx.z;
  const int g = H / Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  __shared__ float sq[kMaxGroup][D];
  __shared__ float sm[kAttnWarps][kMaxGroup], sl[kAttnWarps][kMaxGroup];
  __shared__ float so[kAttnWarps][kMaxGroup][D];
  __shared__ unsigned int s_ticket;

  pdl_wait();
  const int L = pos_for_len ? pos_for_len[b] + 1 : kv_len[b];
  const bool valid = L >= 1 && L <= cap;
  const int t0 = s * ch;
  const int t1 = valid ? min(L, t0 + ch) : 0;

  for (int i = threadIdx.x; i < g * D; i += blockDim.x)
    sq[i / D][i % D] = q[((size_t)b * H + kv * g + i / D) * D + i % D] * scale;
  __syncthreads();

  float m[kMaxGroup], l[kMaxGroup], o[kMaxGroup][VPL], qr[kMaxGroup][VPL];
#pragma unroll
  for (int h = 0; h < kMaxGroup; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      o[h][i] = 0.f;
      qr[h][i] = h < g ? sq[h][lane * VPL + i] : 0.f;
    }
  }

  const size_t head_base = ((size_t)b * Hkv + kv) * cap;
  for (int t = t0 + warp; t < t1; t += kAttnWarps) {
    const uint16_t* kr = kc + (head_base + t) * D + lane * VPL;
    const uint16_t* vr = vc + (head_base + t) * D + lane * VPL;
    float kf[VPL], vf[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      kf[i] = bf16_bits_to_f32(kr[i]);
      vf[i] = bf16_bits_to_f32(vr[i]);
    }
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) {
      if (h < g) {
        float d = 0.f;
#pragma unroll
        for (int i = 0; i < VPL; ++i) d = fmaf(qr[h][i], kf[i], d);
        d = warp_sum(d);
        const float mn = fmaxf(m[h], d);
        const float a = expf(m[h] - mn);
        const float p = expf(d - mn);
        l[h] = l[h] * a + p;
#pragma unroll
        for (int i = 0; i < VPL; ++i) o[h][i] = fmaf(o[h][i], a, p * vf[i]);
        m[h] = mn;
      }
    }
  }
  pdl_trigger();

  // merge the warps of this CTA
#pragma unroll
  for (int h = 0; h < kMaxGroup; ++h) {
    if (h < g) {
      if (lane == 0) { sm[warp][h] = m[h]; sl[warp][h] = l[h]; }
#pragma unroll
      for (int i = 0; i < VPL; ++i) so[warp][h][lane * VPL + i] = o[h][i];
    }
  }
  __syncthreads();
  const size_t part = ((size_t)b * H + kv * g) * nsplit;  // + h * nsplit + s
  for (int i = threadIdx.x; i < g * D; i += blockDim.x) {
    const int h = i / D, d = i % D;
    float M = -INFINITY;
    for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, sm[w][h]);
    float Lsum = 0.f, O = 0.f;
    for (int w = 0; w < kAttnWarps; ++w) {
      const float e = sm[w][h] == -INFINITY ? 0.f : expf(sm[w][h] - M);
      Lsum = fmaf(sl[w][h], e, Lsum);
      O = fmaf(so[w][h][d], e, O);
    }
    const size_t pi = part + (size_t)h * nsplit + s;
    ws_o[pi * D + d] = O;
    if (d == 0) {
      ws_ml[pi * 2 + 0] = M;
      ws_ml[pi * 2 + 1] = Lsum;
    }
  }

  // ticket: the last split CTA of this (b, kv) merges all splits
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_ticket = atomicAdd(&ws_cnt[b * Hkv + kv], 1u);
  __syncthreads();
  if (s_ticket != (unsigned)(nsplit - 1)) return;
  __threadfence();

  for (int i = threadIdx.x; i < g * D; i += blockDim.x) {
    const int h = i / D, d = i % D;
    const size_t pb = part + (size_t)h * nsplit;
    float M = -INFINITY;
    for (int j = 0; j < nsplit; ++j) M = fmaxf(M, __ldcg(ws_ml + (pb + j) * 2));
    float Lsum = 0.f, O = 0.f;
    if (M != -INFINITY) {
      for (int j = 0; j < nsplit; ++j) {
        const float mj = __ldcg(ws_ml + (pb + j) * 2);
        const float e = mj == -INFINITY ? 0.f : expf(mj - M);
        Lsum = fmaf(__ldcg(ws_ml + (pb + j) * 2 + 1), e, Lsum);
        O = fmaf(__ldcg(ws_o + (pb + j) * D + d), e, O);
      }
    }
    const float r = (valid && Lsum > 0.f) ? O / Lsum : 0.f;
    const size_t oi = ((size_t)b * H + kv * g + h) * D + d;
    if (out_bf16)
      reinterpret_cast<uint16_t*>(out)[oi] = f32_to_bf16_bits(r);
    else
      reinterpret_cast<float*>(out)[oi] = r;
  }
  if (threadIdx.x == 0) ws_cnt[b * Hkv + kv] = 0u;  // ready for the next launch
}

cudaError_t attention_launch(const float* q, const uint16_t* kc, const uint16_t* vc,
                             const int32_t* kv_len, const int32_t* pos_for_len, void* out,
                             bool out_bf16, int B, int H, int Hkv, int D, int cap, float scale,
                             void* ws, cudaStream_t st, bool pdl) {
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
                      ws_o, ws_ml, ws_cnt);
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
