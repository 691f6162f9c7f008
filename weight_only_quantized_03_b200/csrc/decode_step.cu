// One Qwen3 decode step for B independent sequences.
//
// Op order: turbospark-runtime 0.3.0, src/qwen3_asr_metal.rs, `step`:
// input norm -> q, k, v -> per-head q/k norm -> NeoX RoPE on q and on k ->
// K/V stored at cache row `position` -> attention over rows [0, position]
// -> o_proj -> residual -> post-attention norm -> gate, up -> SiLU-mul ->
// down -> residual; then the final norm and the tied LM head. The embedding
// row is dequantized from the packed table (embed_row_bytes).
//
// Every launch after the first uses Programmatic Dependent Launch: a GEMV
// issues its first weight loads before waiting for the previous kernel, so
// weight streaming overlaps the previous kernel's tail. Nothing here
// synchronises or allocates, so a step can be captured into a CUDA graph.
#include <cstring>
#include <mutex>
#include <vector>

#include "qg_internal.cuh"

namespace qg {

size_t attention_ws_counter_offset(int B, int H, int Hkv, int D, int cap);

struct StepLayout {
  size_t x, xn, xn2, xnf, q, k, v, xa, attn, gate, up, h, oparts, attn_ws, rope, err, total;
};

static size_t a256(size_t v) { return (v + 255) & ~(size_t)255; }

static StepLayout step_layout(const qg_qwen3_config& c, int B, int cap) {
  StepLayout L;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off += a256(bytes); return o; };
  const size_t qd = (size_t)c.heads * c.head_dim, kd = (size_t)c.kv_heads * c.head_dim;
  // the residual stream heads the workspace
  L.x = take((size_t)B * c.hidden * 4);
  L.xn = take((size_t)B * c.hidden * 2);
  L.xn2 = take((size_t)B * c.hidden * 2);
  L.xnf = take((size_t)B * c.hidden * 2);
  L.q = take((size_t)B * qd * 4);
  L.k = take((size_t)B * kd * 4);
  L.v = take((size_t)B * kd * 4);
  L.xa = take((size_t)B * c.hidden * 4);  // residual stream after o_proj
  L.attn = take((size_t)B * qd * 2);
  L.gate = take((size_t)B * c.ffn * 4);
  L.up = take((size_t)B * c.ffn * 4);
  L.h = take((size_t)B * c.ffn * 2);
  L.oparts = take((size_t)B * c.kv_heads * c.hidden * 4);  // fused o_proj partial rows
  L.attn_ws = take(attention_ws_bytes(B, c.heads, c.kv_heads, c.head_dim, cap));
  L.rope = take((size_t)B * (c.head_dim / 2) * 8);
  L.err = take(256);  // error word of the tensor-core matmuls (batched steps)
  L.total = off;
  return L;
}

// Embedding rows; a sequence with a bad token or position gets NaN. Also
// the step's RoPE table: (cos, sin) of pos * theta^(-2i/D) for the D/2
// pairs of every sequence, angles in double (position 0 for a bad
// sequence, whose outputs are NaN anyway); every layer's attention reads it.
__global__ void step_embed_kernel(const uint32_t* __restrict__ w, const uint16_t* __restrict__ s,
                                  const uint16_t* __restrict__ bi, const int32_t* __restrict__ tok,
                                  const int32_t* __restrict__ pos, float* __restrict__ x, int vocab,
                                  int hidden, int cap, float2* __restrict__ rope, int D,
                                  double theta, const __grid_constant__ Prefetch pf,
                                  TlRec* tl) {
  tl_entry(tl);
  // the first layer's weights and cached rows go to L2 (lane 0 of each warp)
  if ((threadIdx.x & 31) == 0 && (pf.n > 0 || pf.kv.kc)) {
    const unsigned wpb = blockDim.x >> 5;
    issue_prefetch(pf, blockIdx.x * wpb + (threadIdx.x >> 5), gridDim.x * wpb);
  }
  pdl_wait();
  const int b = blockIdx.x;
  const int t = tok[b], p = pos[b];
  const bool ok = t >= 0 && t < vocab && p >= 0 && p < cap;
  for (int i = threadIdx.x; i < D / 2; i += blockDim.x) {
    const double inv_freq = pow(theta, -2.0 * (double)i / (double)D);
    double sd, cd;
    sincos((double)(ok ? p : 0) * inv_freq, &sd, &cd);
    rope[(size_t)b * (D / 2) + i] = make_float2((float)cd, (float)sd);
  }
  float* xr = x + (size_t)b * hidden;
  for (int c = threadIdx.x; c < hidden; c += blockDim.x) {
    if (!ok) {
      xr[c] = __int_as_float(0x7fc00000);
      continue;
    }
    const uint32_t word = w[(size_t)t * (hidden / 4) + c / 4];
    const float q = (float)((word >> (8 * (c % 4))) & 0xFFu);
    const size_t g = (size_t)t * (hidden / 64) + c / 64;
    xr[c] = fmaf(q, bf16_bits_to_f32(s[g]), bf16_bits_to_f32(bi[g]));
  }
  pdl_trigger();
  tl_exit(tl);
}

__global__ void step_silu_mul_kernel(const float* __restrict__ g, const float* __restrict__ u,
                                     uint16_t* __restrict__ out, int n) {
  pdl_wait();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const float z = g[i];
    out[i] = f32_to_bf16_bits(z / (1.0f + expf(-z)) * u[i]);
  }
  pdl_trigger();
}

}  // namespace qg

using namespace qg;

static qg_status validate_matrix(const qg_affine8_matrix& m, const char* name, int layer) {
  QG_REQUIRE(m.w && m.scales && m.biases, QG_ERR_INVALID_ARGUMENT,
             "qg_decode_step: layer %d matrix %s has a null pointer", layer, name);
  QG_REQUIRE(aligned(m.w, 16), QG_ERR_MISALIGNED,
             "qg_decode_step: layer %d matrix %s weights not 16-byte aligned", layer, name);
  QG_REQUIRE(aligned(m.scales, 2) && aligned(m.biases, 2), QG_ERR_MISALIGNED,
             "qg_decode_step: layer %d matrix %s scales/biases misaligned", layer, name);
  return QG_OK;
}

static qg_status validate_cfg(const qg_qwen3_config* c, int B, int cap) {
  QG_REQUIRE(c, QG_ERR_INVALID_ARGUMENT, "qg_decode_step: cfg is NULL");
  QG_REQUIRE(c->hidden > 0 && c->hidden % 64 == 0, QG_ERR_UNSUPPORTED_SHAPE,
             "qg_decode_step: hidden=%d must be a positive multiple of 64", c->hidden);
  QG_REQUIRE(c->layers >= 0, QG_ERR_UNSUPPORTED_SHAPE, "qg_decode_step: layers=%d", c->layers);
  QG_REQUIRE(c->heads >= 1 && c->kv_heads >= 1 && c->heads % c->kv_heads == 0 &&
                 c->heads / c->kv_heads <= 8,
             QG_ERR_UNSUPPORTED_SHAPE,
             "qg_decode_step: heads=%d kv_heads=%d (heads must be a multiple of kv_heads, ratio <= 8)",
             c->heads, c->kv_heads);
  QG_REQUIRE(c->head_dim >= 64 && c->head_dim <= 256 && c->head_dim % 64 == 0,
             QG_ERR_UNSUPPORTED_SHAPE,
             "qg_decode_step: head_dim=%d must be a multiple of 64 in [64, 256]", c->head_dim);
  QG_REQUIRE(((long long)c->heads * c->head_dim) % 64 == 0, QG_ERR_UNSUPPORTED_SHAPE,
             "qg_decode_step: heads*head_dim must be a multiple of 64");
  QG_REQUIRE(c->ffn > 0 && c->ffn % 64 == 0, QG_ERR_UNSUPPORTED_SHAPE,
             "qg_decode_step: ffn=%d must be a positive multiple of 64", c->ffn);
  QG_REQUIRE(c->vocab >= 1, QG_ERR_UNSUPPORTED_SHAPE, "qg_decode_step: vocab=%d", c->vocab);
  QG_REQUIRE(c->eps >= 0.f && c->theta > 0.0, QG_ERR_INVALID_ARGUMENT,
             "qg_decode_step: eps must be >= 0 and theta > 0");
  QG_REQUIRE(B >= 1 && B <= 32, QG_ERR_UNSUPPORTED_SHAPE, "qg_decode_step: B=%d must be in [1, 32]",
             B);
  QG_REQUIRE(cap >= 1, QG_ERR_UNSUPPORTED_SHAPE, "qg_decode_step: cap=%d must be >= 1", cap);
  return QG_OK;
}

extern "C" size_t qg_decode_step_workspace_size(const qg_qwen3_config* cfg, int B, int cap) {
  if (!cfg || B < 1 || cap < 1 || cfg->heads < 1 || cfg->kv_heads < 1) return 0;
  return step_layout(*cfg, B, cap).total;
}

// The step's buffers inside its workspace.
struct StepBufs {
  float* x;
  uint16_t *xn, *xn2, *xnf;
  float *q, *k, *v, *xa;
  uint16_t* attn;
  float *gate, *up;
  uint16_t* hm;
  void* aws;
  float2* rope;
  unsigned* err;
  float* oparts;
};

static StepBufs step_bufs(void* ws, const StepLayout& Ly) {
  uint8_t* base = reinterpret_cast<uint8_t*>(ws);
  StepBufs b;
  b.x = reinterpret_cast<float*>(base + Ly.x);
  b.xn = reinterpret_cast<uint16_t*>(base + Ly.xn);
  b.xn2 = reinterpret_cast<uint16_t*>(base + Ly.xn2);
  b.xnf = reinterpret_cast<uint16_t*>(base + Ly.xnf);
  b.q = reinterpret_cast<float*>(base + Ly.q);
  b.k = reinterpret_cast<float*>(base + Ly.k);
  b.v = reinterpret_cast<float*>(base + Ly.v);
  b.xa = reinterpret_cast<float*>(base + Ly.xa);
  b.attn = reinterpret_cast<uint16_t*>(base + Ly.attn);
  b.gate = reinterpret_cast<float*>(base + Ly.gate);
  b.up = reinterpret_cast<float*>(base + Ly.up);
  b.hm = reinterpret_cast<uint16_t*>(base + Ly.h);
  b.aws = base + Ly.attn_ws;
  b.rope = reinterpret_cast<float2*>(base + Ly.rope);
  b.err = reinterpret_cast<unsigned*>(base + Ly.err);
  b.oparts = reinterpret_cast<float*>(base + Ly.oparts);
  return b;
}

// The decoder layers on the residual stream sb.x (5 launches a layer where
// the tensor-core GEMV takes the shapes), in stream order on s.
// L2 prefetch lists of the step: each kernel hands L2 the data of the
// kernel two launches after it (q/k/v -> o_proj, attention -> gate/up,
// o_proj -> down, gate/up -> the next layer's q/k/v, down -> the next
// layer's cached K/V rows), so the weight stream runs ahead of the chain.
static void pf_matrix(Prefetch& pf, const qg_affine8_matrix& m, int N, int K) {
  if (pf.n + 3 > kMaxPf) return;
  pf.r[pf.n++] = PfRange{m.w, (unsigned long long)N * K};
  pf.r[pf.n++] = PfRange{m.scales, (unsigned long long)N * (K / 64) * 2};
  pf.r[pf.n++] = PfRange{m.biases, (unsigned long long)N * (K / 64) * 2};
}

static Prefetch pf_qkv(const qg_qwen3_config& c, const qg_qwen3_layer& L) {
  Prefetch pf = {};
  const int HD = c.heads * c.head_dim, KD = c.kv_heads * c.head_dim;
  pf_matrix(pf, L.q, HD, c.hidden);
  pf_matrix(pf, L.k, KD, c.hidden);
  pf_matrix(pf, L.v, KD, c.hidden);
  return pf;
}

static Prefetch pf_kv(const qg_qwen3_config& c, const uint16_t* kc, const uint16_t* vc,
                      const int32_t* positions, int B, int cap) {
  Prefetch pf = {};
  pf.kv = KvPf{kc, vc, positions, B, c.kv_heads, cap, c.head_dim};
  return pf;
}

// From this batch size on, the tied LM head (a wave of 128-row tiles or
// more) runs as a tensor-core matmul (gemm_affine8_sm100.cu: the batch rows
// are the MMA's N, each weight tile is dequantized once for all rows) after
// a separate final RMSNorm; the layers' matrices, a few dozen tiles each,
// stay on the tensor-core GEMV with its fused prologues.
constexpr int kStepGemmBatch = 5;

// o_proj folded into the attention kernel (one launch fewer per layer) where
// the shapes allow it: built only with QG_FUSE_OPROJ. Measured on the B200
// (0.6B shape, batch 1, KV 512) the folded attention launch took 21 us
// against 8.5 us for attention plus 4.8 us for the o_proj GEMV, so by
// default o_proj stays a GEMV launch of its own.
#ifdef QG_FUSE_OPROJ
constexpr bool kStepFuseOProj = true;
#else
constexpr bool kStepFuseOProj = false;
#endif

// The tensor-core GEMV can form its input in its prologue (RMSNorm of the
// residual stream, SiLU(gate) * up), which saves a launch per layer at batch
// 1. But every CTA forms all B x K values: measured on the B200 in the
// 1.7B-shaped step at batch 8 (K = 6144 for down), the down GEMV spent 43 us
// after its wait doing so. Past this many values the input is formed once by
// its own kernel (RMSNorm or SiLU-mul, bf16 out) and the GEMV reads it as is.
constexpr long long kFusePrologueMaxBK = 8192;
static bool fuse_prologue(int B, int K) { return (long long)B * K <= kFusePrologueMaxBK; }

static bool head_uses_gemm(const qg_qwen3_config& c, int N, int B) {
  return B >= kStepGemmBatch && c.hidden % 64 == 0 && (N + 127) / 128 >= num_sms();
}

// `after_layer`, when given, is called with the layer index after each
// layer's launches are enqueued.
template <class AfterLayer>
static void enqueue_layers(const qg_qwen3_config& c, const qg_qwen3_layer* layers,
                           uint16_t* k_cache, uint16_t* v_cache, int cap, const int32_t* tokens,
                           const int32_t* positions, int B, const StepBufs& sb, cudaStream_t s,
                           AfterLayer&& after_layer) {
  const int H = c.heads, Hkv = c.kv_heads, D = c.head_dim;
  const size_t layer_cache = (size_t)B * Hkv * cap * D;
  const float scale = 1.0f / sqrtf((float)D);
  float* x = sb.x;
  for (int l = 0; l < c.layers; ++l) {
    const qg_qwen3_layer& L = layers[l];
    uint16_t* kc = k_cache + l * layer_cache;
    uint16_t* vc = v_cache + l * layer_cache;
    GemvSeg qkv[3] = {{L.q.w, L.q.scales, L.q.biases, sb.q, nullptr, H * D, 0},
                      {L.k.w, L.k.scales, L.k.biases, sb.k, nullptr, Hkv * D, 0},
                      {L.v.w, L.v.scales, L.v.biases, sb.v, nullptr, Hkv * D, 0}};
    Prefetch pf_o = {}, pf_gu = {}, pf_dn = {};
    pf_matrix(pf_o, L.o, c.hidden, H * D);
    pf_matrix(pf_gu, L.gate, c.ffn, c.hidden);
    pf_matrix(pf_gu, L.up, c.ffn, c.hidden);
    pf_matrix(pf_dn, L.down, c.hidden, c.ffn);
    const bool last = l + 1 == c.layers;
    const Prefetch pf_next_qkv = last ? Prefetch{} : pf_qkv(c, layers[l + 1]);
    const Prefetch pf_next_kv =
        last ? Prefetch{} : pf_kv(c, kc + layer_cache, vc + layer_cache, positions, B, cap);
    GemvSeg gu_f[2] = {{L.gate.w, L.gate.scales, L.gate.biases, sb.gate, nullptr, c.ffn, 0},
                       {L.up.w, L.up.scales, L.up.biases, sb.up, nullptr, c.ffn, 0}};
    if (kStepFuseOProj && gemv_tc_eligible(qkv, 3, c.hidden, B, false) &&
        gemv_tc_eligible(gu_f, 2, c.hidden, B, false) && aligned(L.o.scales, 8) &&
        aligned(L.o.biases, 8) && attention_oproj_fusable(B, H, Hkv, D, cap, c.hidden)) {
      // 4 launches: q/k/v (input norm in the prologue); attention with o_proj
      // (partial rows per KV head); gate/up with the residual + partials and
      // the post-attention norm in the prologue; down with SiLU-mul
      Prefetch pf_att = {};
      pf_matrix(pf_att, L.gate, c.ffn, c.hidden);
      pf_matrix(pf_att, L.up, c.ffn, c.hidden);
      pf_matrix(pf_att, L.down, c.hidden, c.ffn);
      Prefetch pf_gu2 = pf_next_qkv;
      tl_set_kind(kTlQkv);
      gemv_tc_launch_rmsnorm(qkv, 3, x, L.input_norm, c.eps, c.hidden, B, s, true, sb.xn, &pf_o);
      tl_set_kind(kTlAttn);
      const OProjFuse op = {L.o.w, L.o.scales, L.o.biases, sb.oparts, c.hidden};
      attention_launch_step(sb.q, sb.k, sb.v, L.q_norm, L.k_norm, tokens, c.vocab, c.eps, sb.rope,
                            kc, vc, positions, sb.attn, B, H, Hkv, D, cap, scale, sb.aws, s, true,
                            &pf_att, &op);
      tl_set_kind(kTlGateUp);
      gemv_tc_launch_rmsnorm_parts(gu_f, 2, x, sb.oparts, Hkv, sb.xa, L.post_norm, c.eps,
                                   c.hidden, B, s, true, sb.xn2, &pf_gu2);
      tl_set_kind(kTlDown);
      GemvSeg dn = {L.down.w, L.down.scales, L.down.biases, x, sb.xa, c.hidden, 0};
      gemv_tc_launch_silu_mul(&dn, 1, sb.gate, sb.up, c.ffn, B, s, true, sb.hm, &pf_next_kv);
      after_layer(l);
      continue;
    }
    // RMSNorm and SiLU-mul run in the next GEMV's prologue where the
    // tensor-core GEMV takes the shape, as separate kernels otherwise
    tl_set_kind(kTlQkv);
    if (fuse_prologue(B, c.hidden) && gemv_tc_eligible(qkv, 3, c.hidden, B, false)) {
      gemv_tc_launch_rmsnorm(qkv, 3, x, L.input_norm, c.eps, c.hidden, B, s, true, sb.xn, &pf_o);
    } else {
      rmsnorm_launch(x, L.input_norm, c.eps, sb.xn, true, B, c.hidden, s, true);
      gemv_affine8_launch(qkv, 3, sb.xn, false, c.hidden, B, s, true);
    }
    tl_set_kind(kTlAttn);
    attention_launch_step(sb.q, sb.k, sb.v, L.q_norm, L.k_norm, tokens, c.vocab, c.eps, sb.rope,
                          kc, vc, positions, sb.attn, B, H, Hkv, D, cap, scale, sb.aws, s, true,
                          &pf_gu);
    // o_proj: xa = x + W_o attn; down: x = xa + W_down h (the residual
    // stream after attention stays readable until the next layer)
    GemvSeg o = {L.o.w, L.o.scales, L.o.biases, sb.xa, x, c.hidden, 0};
    tl_set_kind(kTlO);
    if (gemv_tc_eligible(&o, 1, H * D, B, false))
      gemv_tc_launch_pf(&o, 1, sb.attn, H * D, B, s, true, &pf_dn);
    else
      gemv_affine8_launch(&o, 1, sb.attn, false, H * D, B, s, true);
    GemvSeg gu[2] = {{L.gate.w, L.gate.scales, L.gate.biases, sb.gate, nullptr, c.ffn, 0},
                     {L.up.w, L.up.scales, L.up.biases, sb.up, nullptr, c.ffn, 0}};
    tl_set_kind(kTlGateUp);
    if (fuse_prologue(B, c.hidden) && gemv_tc_eligible(gu, 2, c.hidden, B, false)) {
      gemv_tc_launch_rmsnorm(gu, 2, sb.xa, L.post_norm, c.eps, c.hidden, B, s, true, sb.xn2,
                             &pf_next_qkv);
    } else {
      rmsnorm_launch(sb.xa, L.post_norm, c.eps, sb.xn2, true, B, c.hidden, s, true);
      gemv_affine8_launch(gu, 2, sb.xn2, false, c.hidden, B, s, true);
    }
    GemvSeg dn = {L.down.w, L.down.scales, L.down.biases, x, sb.xa, c.hidden, 0};
    tl_set_kind(kTlDown);
    if (fuse_prologue(B, c.ffn) && gemv_tc_eligible(&dn, 1, c.ffn, B, false)) {
      gemv_tc_launch_silu_mul(&dn, 1, sb.gate, sb.up, c.ffn, B, s, true, sb.hm, &pf_next_kv);
    } else {
      const int n = B * c.ffn;
      launch_pdl(step_silu_mul_kernel, dim3((n + 255) / 256), dim3(256), 0, s, true,
                 (const float*)sb.gate, (const float*)sb.up, sb.hm, n);
      gemv_affine8_launch(&dn, 1, sb.hm, false, c.ffn, B, s, true);
    }
    after_layer(l);
  }
  tl_set_kind(kTlOther);
}

static void enqueue_layers(const qg_qwen3_config& c, const qg_qwen3_layer* layers,
                           uint16_t* k_cache, uint16_t* v_cache, int cap, const int32_t* tokens,
                           const int32_t* positions, int B, const StepBufs& sb, cudaStream_t s) {
  enqueue_layers(c, layers, k_cache, v_cache, cap, tokens, positions, B, sb, s, [](int) {});
}

// Final RMSNorm and an output head [N][hidden] on sb.x: logits [B][N].
static void enqueue_head(const qg_qwen3_config& c, const qg_affine8_matrix& head, int N,
                         const uint16_t* final_norm, float* logits, int B, const StepBufs& sb,
                         cudaStream_t s) {
  GemvSeg h = {head.w, head.scales, head.biases, logits, nullptr, N, 0};
  tl_set_kind(kTlHead);
  if (head_uses_gemm(c, N, B)) {
    rmsnorm_launch(sb.x, final_norm, c.eps, sb.xnf, true, B, c.hidden, s, true);
    const A8Seg m = {head.w, head.scales, head.biases, logits, nullptr, N, 0};
    gemm_affine8_launch(&m, 1, sb.xnf, B, c.hidden, sb.err, s, true, nullptr);
  } else if (fuse_prologue(B, c.hidden) && gemv_tc_eligible(&h, 1, c.hidden, B, false)) {
    gemv_tc_launch_rmsnorm(&h, 1, sb.x, final_norm, c.eps, c.hidden, B, s, true);
  } else {
    rmsnorm_launch(sb.x, final_norm, c.eps, sb.xnf, true, B, c.hidden, s, true);
    gemv_affine8_launch(&h, 1, sb.xnf, false, c.hidden, B, s, true);
  }
  tl_set_kind(kTlOther);
}

// Every launch of one step, in stream order on s (the eager path, and what
// a graph recording of a step holds).
static void enqueue_step(const qg_qwen3_config& c, const qg_qwen3_weights* w, uint16_t* k_cache,
                         uint16_t* v_cache, int cap, const int32_t* tokens,
                         const int32_t* positions, float* logits, int B, void* ws,
                         const StepLayout& Ly, cudaStream_t s) {
  const StepBufs sb = step_bufs(ws, Ly);
  const size_t cnt_off = attention_ws_counter_offset(B, c.heads, c.kv_heads, c.head_dim, cap);
  cudaMemsetAsync(reinterpret_cast<uint8_t*>(sb.aws) + cnt_off, 0, (size_t)B * c.kv_heads * 4, s);
  if (head_uses_gemm(c, c.vocab, B)) cudaMemsetAsync(sb.err, 0, 4, s);
  Prefetch pf0 = {};
  if (c.layers > 0) {
    pf0 = pf_qkv(c, w->layers[0]);
    pf0.kv = KvPf{k_cache, v_cache, positions, B, c.kv_heads, cap, c.head_dim};
  }
  launch_pdl(step_embed_kernel, dim3(B), dim3(256), 0, s, true, w->embed.w, w->embed.scales,
             w->embed.biases, tokens, positions, sb.x, c.vocab, c.hidden, cap, sb.rope, c.head_dim,
             c.theta, pf0, tl_take(kTlEmbed));
  enqueue_layers(c, w->layers, k_cache, v_cache, cap, tokens, positions, B, sb, s);
  enqueue_head(c, w->embed, c.vocab, w->final_norm, logits, B, sb, s);
}

// ---------------------------------------------------------------------------
// Step graphs. Launching a step's 5 launches per layer one by one costs host
// time comparable to the step itself, so a call on a non-default stream that
// is not being captured records its launches into a CUDA graph once and
// replays that graph afterwards. The graph holds every pointer and size of
// the call, so it is keyed on all of them, the weight tables' contents
// included (a caller may rewrite its host weight struct in place); any
// difference records a new graph. Up to kMaxGraphs graphs are kept, the
// least recently used is dropped first.
// ---------------------------------------------------------------------------

namespace {

constexpr size_t kMaxGraphs = 8;

struct StepGraph {
  std::vector<uint64_t> key;
  cudaGraphExec_t exec;
  uint64_t used;
};

std::mutex g_graph_mu;
std::vector<StepGraph> g_graphs;
uint64_t g_graph_tick = 0;
bool g_graphs_on = true;

void key_push(std::vector<uint64_t>& k, const void* p) { k.push_back((uint64_t)(uintptr_t)p); }

void key_cfg(std::vector<uint64_t>& k, const qg_qwen3_config& c, int B, int cap) {
  const int ints[] = {c.hidden, c.layers, c.heads, c.kv_heads, c.head_dim, c.ffn, c.vocab, B, cap};
  for (int v : ints) k.push_back((uint64_t)(uint32_t)v);
  uint32_t eps_bits;
  memcpy(&eps_bits, &c.eps, 4);
  uint64_t theta_bits;
  memcpy(&theta_bits, &c.theta, 8);
  k.push_back(eps_bits);
  k.push_back(theta_bits);
}

void key_matrix(std::vector<uint64_t>& k, const qg_affine8_matrix& m) {
  key_push(k, m.w);
  key_push(k, m.scales);
  key_push(k, m.biases);
}

void key_layers(std::vector<uint64_t>& k, const qg_qwen3_layer* layers, int n) {
  for (int l = 0; l < n; ++l) {
    const qg_qwen3_layer& L = layers[l];
    for (const qg_affine8_matrix* m : {&L.q, &L.k, &L.v, &L.o, &L.gate, &L.up, &L.down})
      key_matrix(k, *m);
    for (const void* p : {(const void*)L.input_norm, (const void*)L.post_norm,
                          (const void*)L.q_norm, (const void*)L.k_norm})
      key_push(k, p);
  }
}

std::vector<uint64_t> step_key(const qg_qwen3_config& c, const qg_qwen3_weights* w,
                               const void* kc, const void* vc, int cap, const void* tokens,
                               const void* positions, const void* logits, int B, const void* ws) {
  std::vector<uint64_t> k;
  k.reserve(32 + (size_t)c.layers * 25);
  k.push_back(1);  // what: a decode step
  key_cfg(k, c, B, cap);
  for (const void* p : {kc, vc, tokens, positions, logits, ws}) key_push(k, p);
  key_matrix(k, w->embed);
  key_push(k, w->final_norm);
  key_layers(k, w->layers, c.layers);
  return k;
}

}  // namespace

extern "C" void qg_step_graphs_enable(int on) {
  std::lock_guard<std::mutex> lock(g_graph_mu);
  g_graphs_on = on != 0;
}

extern "C" void qg_step_graphs_clear(void) {
  std::lock_guard<std::mutex> lock(g_graph_mu);
  for (StepGraph& g : g_graphs) cudaGraphExecDestroy(g.exec);
  g_graphs.clear();
}

// Runs `enqueue` on stream s: replayed from a recorded graph keyed on `key`
// when the stream allows it (recorded on first use), launched eagerly
// otherwise or when recording fails.
template <class Enqueue>
static qg_status run_recorded(std::vector<uint64_t> key, cudaStream_t s, Enqueue&& enqueue,
                              const char* what) {
  bool graphs_on;
  {
    std::lock_guard<std::mutex> lock(g_graph_mu);
    graphs_on = g_graphs_on;
  }
  cudaStreamCaptureStatus cap_status = cudaStreamCaptureStatusActive;
  int device = 0;
  if (!graphs_on || s == nullptr || s == cudaStreamLegacy || s == cudaStreamPerThread ||
      cudaStreamIsCapturing(s, &cap_status) != cudaSuccess ||
      cap_status != cudaStreamCaptureStatusNone || cudaGetDevice(&device) != cudaSuccess) {
    cudaGetLastError();
    enqueue();
    return check_launch(what);
  }
  key.push_back((uint64_t)(uint32_t)device);
  {
    std::lock_guard<std::mutex> lock(g_graph_mu);
    for (StepGraph& g : g_graphs) {
      if (g.key == key) {
        g.used = ++g_graph_tick;
        const cudaError_t e = cudaGraphLaunch(g.exec, s);
        if (e != cudaSuccess) {
          set_error("%s: %s", what, cudaGetErrorString(e));
          return QG_ERR_CUDA;
        }
        return QG_OK;
      }
    }
  }
  // record this call's launches, then replay the recording
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  cudaError_t e = cudaStreamBeginCapture(s, cudaStreamCaptureModeThreadLocal);
  if (e == cudaSuccess) {
    enqueue();
    e = cudaStreamEndCapture(s, &graph);
  }
  if (e == cudaSuccess) e = cudaGraphInstantiate(&exec, graph, 0);
  if (graph) cudaGraphDestroy(graph);
  if (e != cudaSuccess) {  // no graph: launch eagerly
    cudaGetLastError();
    if (exec) cudaGraphExecDestroy(exec);
    enqueue();
    return check_launch(what);
  }
  e = cudaGraphLaunch(exec, s);
  {
    std::lock_guard<std::mutex> lock(g_graph_mu);
    if (g_graphs.size() >= kMaxGraphs) {
      size_t lru = 0;
      for (size_t i = 1; i < g_graphs.size(); ++i)
        if (g_graphs[i].used < g_graphs[lru].used) lru = i;
      cudaGraphExecDestroy(g_graphs[lru].exec);
      g_graphs.erase(g_graphs.begin() + lru);
    }
    g_graphs.push_back(StepGraph{std::move(key), exec, ++g_graph_tick});
  }
  if (e != cudaSuccess) {
    set_error("%s: %s", what, cudaGetErrorString(e));
    return QG_ERR_CUDA;
  }
  return QG_OK;
}

extern "C" qg_status qg_decode_step(const qg_qwen3_config* cfg, const qg_qwen3_weights* w,
                                    uint16_t* k_cache, uint16_t* v_cache, int cap,
                                    const int32_t* tokens, const int32_t* positions, float* logits,
                                    int B, void* ws, size_t ws_bytes, void* stream) {
  clear_error();
  qg_status st = validate_cfg(cfg, B, cap);
  if (st != QG_OK) return st;
  const qg_qwen3_config& c = *cfg;
  QG_REQUIRE(w, QG_ERR_INVALID_ARGUMENT, "qg_decode_step: weights is NULL");
  QG_REQUIRE(c.layers == 0 || w->layers, QG_ERR_INVALID_ARGUMENT,
             "qg_decode_step: weights->layers is NULL");
  if ((st = validate_matrix(w->embed, "embed", -1)) != QG_OK) return st;
  QG_REQUIRE(w->final_norm && aligned(w->final_norm, 2), QG_ERR_INVALID_ARGUMENT,
             "qg_decode_step: final_norm is NULL or misaligned");
  for (int l = 0; l < c.layers; ++l) {
    const qg_qwen3_layer& L = w->layers[l];
    const qg_affine8_matrix* ms[7] = {&L.q, &L.k, &L.v, &L.o, &L.gate, &L.up, &L.down};
    const char* names[7] = {"q", "k", "v", "o", "gate", "up", "down"};
    for (int i = 0; i < 7; ++i)
      if ((st = validate_matrix(*ms[i], names[i], l)) != QG_OK) return st;
    QG_REQUIRE(L.input_norm && L.post_norm && L.q_norm && L.k_norm, QG_ERR_INVALID_ARGUMENT,
               "qg_decode_step: layer %d has a null norm weight", l);
  }
  QG_REQUIRE(c.layers == 0 || (k_cache && v_cache), QG_ERR_INVALID_ARGUMENT,
             "qg_decode_step: null k_cache or v_cache");
  QG_REQUIRE(aligned(k_cache, 16) && aligned(v_cache, 16), QG_ERR_MISALIGNED,
             "qg_decode_step: k_cache/v_cache not 16-byte aligned");
  QG_REQUIRE(tokens && positions && logits, QG_ERR_INVALID_ARGUMENT,
             "qg_decode_step: null tokens, positions or logits");
  QG_REQUIRE(aligned(tokens, 4) && aligned(positions, 4) && aligned(logits, 4), QG_ERR_MISALIGNED,
             "qg_decode_step: tokens/positions/logits misaligned");
  const StepLayout Ly = step_layout(c, B, cap);
  QG_REQUIRE(ws && ws_bytes >= Ly.total, QG_ERR_WORKSPACE_TOO_SMALL,
             "qg_decode_step: workspace of %zu bytes given, %zu needed", ws_bytes, Ly.total);
  QG_REQUIRE(aligned(ws, 256), QG_ERR_MISALIGNED, "qg_decode_step: ws not 256-byte aligned");

  cudaStream_t s = (cudaStream_t)stream;
  return run_recorded(step_key(c, w, k_cache, v_cache, cap, tokens, positions, logits, B, ws), s,
                      [&] {
                        enqueue_step(c, w, k_cache, v_cache, cap, tokens, positions, logits, B,
                                     ws, Ly, s);
                      },
                      "qg_decode_step");
}

extern "C" qg_status qg_decode_step_inspect(const qg_qwen3_config* cfg, int B, int cap,
                                           size_t offsets[4]) {
  clear_error();
  qg_status st = validate_cfg(cfg, B, cap);
  if (st != QG_OK) return st;
  QG_REQUIRE(offsets, QG_ERR_INVALID_ARGUMENT, "qg_decode_step_inspect: null offsets");
  const StepLayout Ly = step_layout(*cfg, B, cap);
  offsets[0] = Ly.xn;
  offsets[1] = Ly.attn;
  offsets[2] = Ly.xn2;
  offsets[3] = Ly.h;
  return QG_OK;
}

extern "C" qg_status qg_decode_step_inspect_f32(const qg_qwen3_config* cfg, int B, int cap,
                                               size_t offsets[6]) {
  clear_error();
  qg_status st = validate_cfg(cfg, B, cap);
  if (st != QG_OK) return st;
  QG_REQUIRE(offsets, QG_ERR_INVALID_ARGUMENT, "qg_decode_step_inspect_f32: null offsets");
  const StepLayout Ly = step_layout(*cfg, B, cap);
  offsets[0] = Ly.q;
  offsets[1] = Ly.k;
  offsets[2] = Ly.v;
  offsets[3] = Ly.xa;
  offsets[4] = Ly.gate;
  offsets[5] = Ly.up;
  return QG_OK;
}

// ---------------------------------------------------------------------------
// Code predictor: makima src/tts/qwen3/code_predictor.rs, CodePredictor::
// predict. Per group g = 1 .. groups-1: embed code g-1 with table g-1,
// concatenate it after the main model's hidden state, project with
// input_proj, run the layers (each with a fresh KV cache: one row at
// position 0), final norm, head g, greedy code. The concatenated input is a
// GEMV input and is stored as bf16, like every activation that feeds a GEMV
// in this library.
// ---------------------------------------------------------------------------

namespace qg {

// codes[0] = code0 and every sequence's position 0; the RoPE table of
// position 0 (all angles 0).
__global__ void cp_start_kernel(const int32_t* __restrict__ code0, int32_t* __restrict__ codes0,
                                int32_t* __restrict__ pos, float2* __restrict__ rope, int D) {
  pdl_wait();
  const int b = blockIdx.x;
  if (threadIdx.x == 0) {
    codes0[b] = code0[b];
    pos[b] = 0;
  }
  for (int i = threadIdx.x; i < D / 2; i += blockDim.x)
    rope[(size_t)b * (D / 2) + i] = make_float2(1.0f, 0.0f);
}

// bf16(concat(lm_hidden[b], embed(prev[b]))) [B][2 hidden]; an out-of-range
// code gives NaN in its half.
__global__ void cp_input_kernel(const float* __restrict__ lm_hidden, const uint32_t* __restrict__ ew,
                                const uint16_t* __restrict__ es, const uint16_t* __restrict__ eb,
                                const int32_t* __restrict__ prev, uint16_t* __restrict__ out,
                                int hidden, int vocab) {
  pdl_wait();
  const int b = blockIdx.x;
  const int t = __ldcg(prev + b);
  const bool ok = t >= 0 && t < vocab;
  uint16_t* o = out + (size_t)b * 2 * hidden;
  for (int c = threadIdx.x; c < hidden; c += blockDim.x) {
    o[c] = f32_to_bf16_bits(__ldcg(lm_hidden + (size_t)b * hidden + c));
    float e = __int_as_float(0x7fc00000);
    if (ok) {
      const uint32_t word = ew[(size_t)t * (hidden / 4) + c / 4];
      const float q = (float)((word >> (8 * (c % 4))) & 0xFFu);
      const size_t g = (size_t)t * (hidden / 64) + c / 64;
      e = fmaf(q, bf16_bits_to_f32(es[g]), bf16_bits_to_f32(eb[g]));
    }
    o[hidden + c] = f32_to_bf16_bits(e);
  }
}

}  // namespace qg

namespace {

struct CpLayout {
  StepLayout step;  // the step's buffers for cap = 1 (from offset 0)
  size_t comb, kc, vc, pos, am, logits, total;
};

CpLayout cp_layout(const qg_qwen3_config& c, int B) {
  CpLayout L;
  L.step = step_layout(c, B, 1);
  size_t off = L.step.total;
  auto take = [&](size_t bytes) { size_t o = off; off += (bytes + 255) & ~(size_t)255; return o; };
  const size_t cache = (size_t)c.layers * B * c.kv_heads * 1 * c.head_dim * 2;
  L.comb = take((size_t)B * 2 * c.hidden * 2);
  L.kc = take(cache);
  L.vc = take(cache);
  L.pos = take((size_t)B * 4);
  L.am = take(argmax_ws_bytes(B, c.vocab));
  L.logits = take((size_t)B * c.vocab * 4);
  L.total = off;
  return L;
}

}  // namespace

extern "C" size_t qg_code_predict_workspace_size(const qg_qwen3_config* cfg, int B) {
  if (!cfg || B < 1 || cfg->heads < 1 || cfg->kv_heads < 1 || cfg->vocab < 1) return 0;
  return cp_layout(*cfg, B).total;
}

namespace {

// Trace of a traced code prediction: per group g = 1 .. groups-1, the bf16
// concatenated input, then one slot after input_proj and one after each
// layer, each a copy of the workspace head (the step buffers up to the
// attention scratch) followed by the K and V rows the slot's layer wrote.
struct CpTrace {
  size_t comb, snap, kv, slot, group, total;
};

CpTrace cp_trace_layout(const qg_qwen3_config& c, int B, int groups) {
  const CpLayout Ly = cp_layout(c, B);
  CpTrace T;
  T.comb = a256((size_t)B * 2 * c.hidden * 2);
  T.snap = Ly.step.attn_ws;  // x .. h: every step buffer before the attention scratch
  T.kv = a256((size_t)B * c.kv_heads * c.head_dim * 2);
  T.slot = T.snap + 2 * T.kv;
  T.group = T.comb + (size_t)(c.layers + 1) * T.slot;
  T.total = (size_t)(groups > 1 ? groups - 1 : 0) * T.group;
  return T;
}

qg_status code_predict_impl(const qg_qwen3_config* cfg, const qg_code_predictor_weights* w,
                            const float* lm_hidden, const int32_t* code0, int32_t* codes,
                            float* logits, int B, void* ws, size_t ws_bytes, void* trace,
                            size_t trace_bytes, void* stream, const char* what) {
  clear_error();
  qg_status st = validate_cfg(cfg, B, 1);
  if (st != QG_OK) return st;
  const qg_qwen3_config& c = *cfg;
  QG_REQUIRE(w, QG_ERR_INVALID_ARGUMENT, "%s: weights is NULL", what);
  QG_REQUIRE(w->groups >= 2 && w->groups <= 64, QG_ERR_UNSUPPORTED_SHAPE,
             "%s: groups=%d must be in [2, 64]", what, w->groups);
  QG_REQUIRE(w->code_embed && w->heads && w->final_norm && (c.layers == 0 || w->layers),
             QG_ERR_INVALID_ARGUMENT, "%s: null table, head, norm or layer array", what);
  if ((st = validate_matrix(w->input_proj, "input_proj", -1)) != QG_OK) return st;
  for (int g = 1; g < w->groups; ++g) {
    if ((st = validate_matrix(w->code_embed[g - 1], "code_embed", g - 1)) != QG_OK) return st;
    if ((st = validate_matrix(w->heads[g], "heads", g)) != QG_OK) return st;
  }
  for (int l = 0; l < c.layers; ++l) {
    const qg_qwen3_layer& L = w->layers[l];
    for (const qg_affine8_matrix* m : {&L.q, &L.k, &L.v, &L.o, &L.gate, &L.up, &L.down})
      if ((st = validate_matrix(*m, "layer", l)) != QG_OK) return st;
    QG_REQUIRE(L.input_norm && L.post_norm && L.q_norm && L.k_norm, QG_ERR_INVALID_ARGUMENT,
               "%s: layer %d has a null norm weight", what, l);
  }
  QG_REQUIRE(lm_hidden && code0 && codes, QG_ERR_INVALID_ARGUMENT,
             "%s: null lm_hidden, code0 or codes", what);
  QG_REQUIRE(aligned(lm_hidden, 4) && aligned(code0, 4) && aligned(codes, 4) &&
                 aligned(logits, 4),
             QG_ERR_MISALIGNED, "%s: lm_hidden/code0/codes/logits misaligned", what);
  const CpLayout Ly = cp_layout(c, B);
  QG_REQUIRE(ws && ws_bytes >= Ly.total, QG_ERR_WORKSPACE_TOO_SMALL,
             "%s: workspace of %zu bytes given, %zu needed", what, ws_bytes, Ly.total);
  QG_REQUIRE(aligned(ws, 256), QG_ERR_MISALIGNED, "%s: ws not 256-byte aligned", what);
  const CpTrace T = cp_trace_layout(c, B, w->groups);
  if (trace) {
    QG_REQUIRE(trace_bytes >= T.total, QG_ERR_WORKSPACE_TOO_SMALL,
               "%s: trace of %zu bytes given, %zu needed", what, trace_bytes, T.total);
    QG_REQUIRE(aligned(trace, 256), QG_ERR_MISALIGNED, "%s: trace not 256-byte aligned", what);
  }

  cudaStream_t s = (cudaStream_t)stream;
  uint8_t* base = reinterpret_cast<uint8_t*>(ws);
  uint8_t* tr = reinterpret_cast<uint8_t*>(trace);
  const size_t kv_row = (size_t)B * c.kv_heads * c.head_dim * 2;  // one layer's cache (cap 1)
  auto enqueue = [&] {
    const StepBufs sb = step_bufs(ws, Ly.step);
    uint16_t* comb = reinterpret_cast<uint16_t*>(base + Ly.comb);
    uint16_t* kc = reinterpret_cast<uint16_t*>(base + Ly.kc);
    uint16_t* vc = reinterpret_cast<uint16_t*>(base + Ly.vc);
    int32_t* pos = reinterpret_cast<int32_t*>(base + Ly.pos);
    void* am = base + Ly.am;
    const size_t cnt_off = attention_ws_counter_offset(B, c.heads, c.kv_heads, c.head_dim, 1);
    cudaMemsetAsync(reinterpret_cast<uint8_t*>(sb.aws) + cnt_off, 0, (size_t)B * c.kv_heads * 4,
                    s);
    launch_pdl(cp_start_kernel, dim3(B), dim3(64), 0, s, true, code0, codes, pos, sb.rope,
               c.head_dim);
    for (int g = 1; g < w->groups; ++g) {
      const int32_t* prev = codes + (size_t)(g - 1) * B;
      const qg_affine8_matrix& E = w->code_embed[g - 1];
      launch_pdl(cp_input_kernel, dim3(B), dim3(256), 0, s, true, lm_hidden, E.w, E.scales,
                 E.biases, prev, comb, c.hidden, c.vocab);
      GemvSeg ip = {w->input_proj.w, w->input_proj.scales, w->input_proj.biases, sb.x, nullptr,
                    c.hidden, 0};
      gemv_affine8_launch(&ip, 1, comb, false, 2 * c.hidden, B, s, true);
      uint8_t* tg = tr ? tr + (size_t)(g - 1) * T.group : nullptr;
      auto snapshot = [&](int slot) {
        uint8_t* d = tg + T.comb + (size_t)slot * T.slot;
        cudaMemcpyAsync(d, base, T.snap, cudaMemcpyDeviceToDevice, s);
        if (slot > 0) {
          const size_t lo = (size_t)(slot - 1) * kv_row;
          cudaMemcpyAsync(d + T.snap, reinterpret_cast<uint8_t*>(kc) + lo, kv_row,
                          cudaMemcpyDeviceToDevice, s);
          cudaMemcpyAsync(d + T.snap + T.kv, reinterpret_cast<uint8_t*>(vc) + lo, kv_row,
                          cudaMemcpyDeviceToDevice, s);
        }
      };
      if (tg) {
        cudaMemcpyAsync(tg, comb, (size_t)B * 2 * c.hidden * 2, cudaMemcpyDeviceToDevice, s);
        snapshot(0);
      }
      enqueue_layers(c, w->layers, kc, vc, 1, prev, pos, B, sb, s, [&](int l) {
        if (tg) snapshot(l + 1);
      });
      float* lg = logits ? logits + (size_t)g * B * c.vocab
                         : reinterpret_cast<float*>(base + Ly.logits);
      enqueue_head(c, w->heads[g], c.vocab, w->final_norm, lg, B, sb, s);
      argmax_launch(lg, B, c.vocab, codes + (size_t)g * B, am, s, true);
    }
  };
  std::vector<uint64_t> key;
  key.push_back(2);  // what: a code prediction
  key_cfg(key, c, B, 1);
  for (const void* p : {(const void*)lm_hidden, (const void*)code0, (const void*)codes,
                        (const void*)logits, (const void*)ws, (const void*)w->final_norm,
                        (const void*)trace})
    key_push(key, p);
  key.push_back((uint64_t)w->groups);
  key_matrix(key, w->input_proj);
  for (int g = 0; g < w->groups; ++g) {
    if (g >= 1) key_matrix(key, w->code_embed[g - 1]);
    if (g >= 1) key_matrix(key, w->heads[g]);
  }
  key_layers(key, w->layers, c.layers);
  return run_recorded(std::move(key), s, enqueue, what);
}

}  // namespace

extern "C" qg_status qg_code_predict(const qg_qwen3_config* cfg, const qg_code_predictor_weights* w,
                                     const float* lm_hidden, const int32_t* code0, int32_t* codes,
                                     float* logits, int B, void* ws, size_t ws_bytes,
                                     void* stream) {
  return code_predict_impl(cfg, w, lm_hidden, code0, codes, logits, B, ws, ws_bytes, nullptr, 0,
                           stream, "qg_code_predict");
}

extern "C" qg_status qg_code_predict_trace_layout(const qg_qwen3_config* cfg, int B, int groups,
                                                  size_t out[4]) {
  clear_error();
  qg_status st = validate_cfg(cfg, B, 1);
  if (st != QG_OK) return st;
  QG_REQUIRE(out, QG_ERR_INVALID_ARGUMENT, "qg_code_predict_trace_layout: null out");
  QG_REQUIRE(groups >= 2 && groups <= 64, QG_ERR_UNSUPPORTED_SHAPE,
             "qg_code_predict_trace_layout: groups=%d must be in [2, 64]", groups);
  const CpTrace T = cp_trace_layout(*cfg, B, groups);
  out[0] = T.total;
  out[1] = T.group;
  out[2] = T.comb;
  out[3] = T.slot;
  return QG_OK;
}

extern "C" qg_status qg_code_predict_traced(const qg_qwen3_config* cfg,
                                            const qg_code_predictor_weights* w,
                                            const float* lm_hidden, const int32_t* code0,
                                            int32_t* codes, float* logits, int B, void* ws,
                                            size_t ws_bytes, void* trace, size_t trace_bytes,
                                            void* stream) {
  if (!trace) {
    clear_error();
    set_error("qg_code_predict_traced: trace is NULL");
    return QG_ERR_INVALID_ARGUMENT;
  }
  return code_predict_impl(cfg, w, lm_hidden, code0, codes, logits, B, ws, ws_bytes, trace,
                           trace_bytes, stream, "qg_code_predict_traced");
}
