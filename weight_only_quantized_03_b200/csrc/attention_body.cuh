// Split-softmax GQA decode attention: the per-CTA body of the kernel in
// attention.cu (which describes the design).
#pragma once

#include "qg_internal.cuh"

namespace qg {

constexpr int kMaxGroup = 8;
constexpr int kMergeMax = 1024;  // (head, split) pairs the last CTA merges from shared memory

// Decode-step fusion: the per-head RMSNorm and NeoX RoPE of q and k and the
// K/V append at the current position (turbospark-runtime 0.3.0,
// src/qwen3_asr_metal.rs, `step`: encode_rms_norm_bf16w_perhead,
// encode_rope_neox_subdim, the cache writes; makima src/tts/qwen3/model.rs,
// apply_head_norm and RotaryEmbedding) run inside the attention kernel.
struct AttnFuse {
  int on;
  const float* k;        // raw k [B][Hkv][D] fp32
  const float* v;        // raw v [B][Hkv][D] fp32
  const uint16_t* qn;    // q_norm weight bf16 [D]
  const uint16_t* kn;    // k_norm weight bf16 [D]
  const int32_t* tok;    // [B]: a bad token writes nothing to the cache
  int vocab;
  float eps;
  const float2* rope;    // (cos, sin) [B][D/2] of the step's positions
  Prefetch pf;           // L2 prefetch work for a later kernel of the step
  TlRec* tl;             // timeline record of this launch, or null
  // o_proj fused into the cluster kernel (ow non-null): each CTA of the
  // cluster of (b, kv) multiplies rows [rank * R, rank * R + R) of W_o's
  // columns of this KV head's query heads by their (bf16) attention output
  // and writes the partial rows to opart[b][kv][hidden]; R = hidden / cs.
  const uint8_t* ow;     // codes [hidden][H*D]
  const uint16_t* os;    // bf16 [hidden][H*D/64]
  const uint16_t* ob;
  float* opart;
  int hidden;
};

// The fused step's L2 prefetch, issued by one thread of each CTA at entry.
__device__ __forceinline__ void attn_issue_prefetch(const AttnFuse& fz) {
  if (fz.on && threadIdx.x == 0 && (fz.pf.n > 0 || fz.pf.kv.kc)) {
    const unsigned cta = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
    issue_prefetch(fz.pf, cta, gridDim.x * gridDim.y * gridDim.z);
  }
}

// q, k, v and the RoPE table are produced by the previous kernels of the
// step; they are read through L2 (ld.global.cg), not kept in L1.
// RMSNorm of one head row src[0..D) with weight w, then the NeoX rotation
// with the (cos, sin) pairs cs[0..D/2); lane owns the pairs (i, i + D/2) for
// i = lane + 32 j. Writes the rotated fp32 values through `put(i, value)`.
// The table is read through L2 (it is written by an earlier kernel) unless
// kSharedCs, when it sits in this CTA's shared memory.
template <bool kSharedCs = false, typename Put>
__device__ __forceinline__ void norm_rope_head(const float* src, const uint16_t* w, int D, float eps,
                                               const float2* cs, int lane, Put put) {
  const int half = D >> 1;
  // the row, its norm weights and its (cos, sin) pairs in one round of loads
  float x1[4], x2[4], w1[4], w2[4];
  float2 r[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int i = lane + 32 * j;
    const bool in = i < half;
    x1[j] = in ? __ldcg(src + i) : 0.f;
    x2[j] = in ? __ldcg(src + i + half) : 0.f;
    w1[j] = in ? bf16_bits_to_f32(w[i]) : 0.f;
    w2[j] = in ? bf16_bits_to_f32(w[i + half]) : 0.f;
    r[j] = in ? (kSharedCs ? cs[i] : __ldcg(cs + i)) : make_float2(0.f, 0.f);
  }
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < 4; ++j) ss = fmaf(x1[j], x1[j], fmaf(x2[j], x2[j], ss));
  ss = warp_sum(ss);
  const float inv = 1.0f / sqrtf(ss / (float)D + eps);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int i = lane + 32 * j;
    if (i >= half) break;
    const float a = x1[j] * inv * w1[j];
    const float c2 = x2[j] * inv * w2[j];
    put(i, a * r[j].x - c2 * r[j].y);
    put(i + half, c2 * r[j].x + a * r[j].y);
  }
}

// VPL consecutive bf16 values (one lane's share of a head row) as fp32, in
// 32-bit words when VPL is even (the row offset lane * VPL is then 4-byte
// aligned). Plain (coherent) loads: in the decode step the kernel itself
// writes the row at the current position before reading it.
template <int VPL>
__device__ __forceinline__ void load_bf16_row(const uint16_t* p, float (&out)[VPL]) {
  if constexpr (VPL % 2 == 0) {
#pragma unroll
    for (int i = 0; i < VPL / 2; ++i) {
      const uint32_t w = reinterpret_cast<const unsigned int*>(p)[i];
      out[2 * i] = bf16_lo(w);
      out[2 * i + 1] = bf16_hi(w);
    }
  } else {
#pragma unroll
    for (int i = 0; i < VPL; ++i) out[i] = bf16_bits_to_f32(p[i]);
  }
}

// One split of one (sequence, kv head): the CTA of NW warps scores rows
// [s*ch, (s+1)*ch) of kv head kv for its g <= GM query heads, leaves the
// split's (max, sum, weighted V) in the workspace, and the last split of the
// pair to finish (atomic ticket) merges all splits in split order. VPL =
// values of a head row per lane (D = 32 VPL). `wait()` runs after the
// first batch of cached rows is in flight and before anything written
// upstream is read (the programmatic-dependent-launch wait).
// The CTA's threads must all call this together; it uses __syncthreads.
template <int VPL, int NW, int GM, class Wait>
__device__ __forceinline__ void attention_body(
    const float* q, const uint16_t* kc, const uint16_t* vc,
    const int32_t* __restrict__ kv_len, const int32_t* __restrict__ pos_for_len,
    void* __restrict__ out, int out_bf16, int H, int Hkv, int cap, float scale, int ch,
    int nsplit, float* __restrict__ ws_o, float* __restrict__ ws_ml,
    unsigned int* __restrict__ ws_cnt, const AttnFuse& fz, int s, int kv, int b, Wait&& wait) {
  constexpr int D = 32 * VPL;
  constexpr int kAttnWarps = NW, kMaxGroup = GM;
  const int g = H / Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  tl_entry(fz.tl);
  attn_issue_prefetch(fz);

  __shared__ float sq[kMaxGroup][D];
  __shared__ float sm[kAttnWarps][kMaxGroup], sl[kAttnWarps][kMaxGroup];
  __shared__ float so[kAttnWarps][kMaxGroup][D];
  __shared__ unsigned int s_ticket;
  // after the warp merge, `so` is free: the split merge reuses it
  constexpr int kMerge = kAttnWarps * kMaxGroup * D / 2 < kMergeMax ? kAttnWarps * kMaxGroup * D / 2
                                                                     : kMergeMax;
  float* s_m = &so[0][0][0];
  float* s_l = s_m + kMerge;

  const int t0 = s * ch;
  const size_t head_base = ((size_t)b * Hkv + kv) * cap;
  // RB rows per warp in flight: all their K/V loads are issued before the
  // first score, so the rows' memory latencies overlap
  constexpr int RB = NW >= 16 ? 2 : (VPL <= 4 ? 8 : 4);
  float kf[RB][VPL], vf[RB][VPL];
#pragma unroll
  for (int r = 0; r < RB; ++r)
#pragma unroll
    for (int i = 0; i < VPL; ++i) kf[r][i] = vf[r][i] = 0.f;
  // Decode step: the positions are an input of the step (final before its
  // first kernel ran), and the cached rows below the position were written
  // by earlier steps, so the first batch of rows is fetched before waiting
  // for the previous kernel; the row at the position is this step's own.
  int pre_p = -1;
  if (fz.on) {
    const int p = pos_for_len[b];
    if (p >= 0 && p < cap) {
      pre_p = p;
      const int t1p = min(p + 1, t0 + ch);
#pragma unroll
      for (int r = 0; r < RB; ++r) {
        const int t = t0 + warp + r * kAttnWarps;
        if (t < t1p && t != p) {
          load_bf16_row<VPL>(kc + (head_base + t) * D + lane * VPL, kf[r]);
          load_bf16_row<VPL>(vc + (head_base + t) * D + lane * VPL, vf[r]);
        }
      }
    }
  }
  wait();
  const int L = pos_for_len ? pos_for_len[b] + 1 : kv_len[b];
  const bool valid = L >= 1 && L <= cap;
  const int t1 = valid ? min(L, t0 + ch) : 0;

  if (!fz.on) {
    for (int i = threadIdx.x; i < g * D; i += blockDim.x)
      sq[i / D][i % D] = __ldcg(q + ((size_t)b * H + kv * g + i / D) * D + i % D) * scale;
  } else {
    // q heads: norm + rope into shared memory (every split recomputes its
    // own); the split holding row p also norms + ropes k and appends k, v
    const int p = pos_for_len[b], tk = fz.tok[b];
    const bool pos_ok = p >= 0 && p < cap && tk >= 0 && tk < fz.vocab;
    const int pr = pos_ok ? p : 0;
    const float2* cs = fz.rope + (size_t)b * (D / 2);
    const bool owner = pos_ok && p >= t0 && p < t0 + ch;
    const size_t row = (((size_t)b * Hkv + kv) * cap + pr) * D;
    for (int hh = warp; hh < g + 2; hh += kAttnWarps) {
      if (hh < g) {
        float* dst = sq[hh];
        norm_rope_head(q + ((size_t)b * H + kv * g + hh) * D, fz.qn, D, fz.eps, cs, lane,
                       [&](int i, float r) { dst[i] = r * scale; });
      } else if (hh == g) {
        if (owner) {
          uint16_t* kdst = const_cast<uint16_t*>(kc) + row;
          norm_rope_head(fz.k + ((size_t)b * Hkv + kv) * D, fz.kn, D, fz.eps, cs, lane,
                         [&](int i, float r) { kdst[i] = f32_to_bf16_bits(r); });
        }
      } else if (owner) {
        uint16_t* vdst = const_cast<uint16_t*>(vc) + row;
        const float* vs = fz.v + ((size_t)b * Hkv + kv) * D;
        for (int d = lane; d < D; d += 32) vdst[d] = f32_to_bf16_bits(__ldcg(vs + d));
      }
    }
  }
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

  for (int tb = t0 + warp; tb < t1; tb += kAttnWarps * RB) {
    // the first batch was fetched before the wait except the current row
    const bool prefetched = pre_p >= 0 && tb == t0 + warp;
#pragma unroll
    for (int r = 0; r < RB; ++r) {
      const int t = tb + r * kAttnWarps;
      if (t < t1 && (!prefetched || t == pre_p)) {
        load_bf16_row<VPL>(kc + (head_base + t) * D + lane * VPL, kf[r]);
        load_bf16_row<VPL>(vc + (head_base + t) * D + lane * VPL, vf[r]);
      }
    }
    // per head: the batch's scores (dot products and warp reductions are
    // independent, so their latencies overlap), then one online-softmax
    // update for the whole batch: running max over the batch, one rescale
    // of (l, o), and the batch's exp-weighted V rows added
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) {
      if (h < g) {
        float dsc[RB];
#pragma unroll
        for (int r = 0; r < RB; ++r) {
          float d = 0.f;
#pragma unroll
          for (int i = 0; i < VPL; ++i) d = fmaf(qr[h][i], kf[r][i], d);
          dsc[r] = d;
        }
#pragma unroll
        for (int r = 0; r < RB; ++r) dsc[r] = warp_sum(dsc[r]);
        float mx = m[h];
#pragma unroll
        for (int r = 0; r < RB; ++r)
          if (tb + r * kAttnWarps < t1) mx = fmaxf(mx, dsc[r]);
        const float a = expf(m[h] - mx);  // 0 while m is still -inf
        l[h] *= a;
#pragma unroll
        for (int i = 0; i < VPL; ++i) o[h][i] *= a;
#pragma unroll
        for (int r = 0; r < RB; ++r) {
          if (tb + r * kAttnWarps < t1) {
            const float p = expf(dsc[r] - mx);
            l[h] += p;
#pragma unroll
            for (int i = 0; i < VPL; ++i) o[h][i] = fmaf(p, vf[r][i], o[h][i]);
          }
        }
        m[h] = mx;
      }
    }
  }

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
  if (s_ticket != (unsigned)(nsplit - 1)) {
    tl_exit(fz.tl);
    return;
  }
  __threadfence();

  auto store_out = [&](int h, int d, float r) {
    const size_t oi = ((size_t)b * H + kv * g + h) * D + d;
    if (out_bf16)
      reinterpret_cast<uint16_t*>(out)[oi] = f32_to_bf16_bits(r);
    else
      reinterpret_cast<float*>(out)[oi] = r;
  };
  const int nw = g * nsplit;
  if (nw <= kMerge) {
    // 1) every split's (max, sum) of the kv head's query heads: one round of
    // loads; 2) per head, the weight of split j, exp(m_j - M) / L (0 for an
    // empty split or an invalid length); 3) the weighted sum of the split
    // outputs, with the loads of several splits in flight together
    for (int i = threadIdx.x; i < nw; i += blockDim.x) {
      s_m[i] = __ldcg(ws_ml + (part + i) * 2);
      s_l[i] = __ldcg(ws_ml + (part + i) * 2 + 1);
    }
    __syncthreads();
    for (int h = warp; h < g; h += kAttnWarps) {
      float M = -INFINITY;
      for (int j = lane; j < nsplit; j += 32) M = fmaxf(M, s_m[h * nsplit + j]);
      M = warp_max(M);
      float Lsum = 0.f;
      for (int j = lane; j < nsplit; j += 32) {
        const float mj = s_m[h * nsplit + j];
        Lsum += (mj == -INFINITY) ? 0.f : s_l[h * nsplit + j] * expf(mj - M);
      }
      Lsum = warp_sum(Lsum);
      const float scale_out = (valid && Lsum > 0.f) ? 1.0f / Lsum : 0.f;
      for (int j = lane; j < nsplit; j += 32) {
        const float mj = s_m[h * nsplit + j];
        s_m[h * nsplit + j] = (mj == -INFINITY) ? 0.f : expf(mj - M) * scale_out;
      }
    }
    __syncthreads();
    for (int i0 = threadIdx.x; i0 < g * D; i0 += 2 * blockDim.x) {
      const int i1 = i0 + blockDim.x;
      const bool has1 = i1 < g * D;
      const int h0 = i0 / D, d0 = i0 % D, h1 = has1 ? i1 / D : h0, d1 = has1 ? i1 % D : d0;
      const float* o0 = ws_o + (part + (size_t)h0 * nsplit) * D + d0;
      const float* o1 = ws_o + (part + (size_t)h1 * nsplit) * D + d1;
      float O0 = 0.f, O1 = 0.f;
#pragma unroll 8
      for (int j = 0; j < nsplit; ++j) {
        O0 = fmaf(s_m[h0 * nsplit + j], __ldcg(o0 + (size_t)j * D), O0);
        O1 = fmaf(s_m[h1 * nsplit + j], __ldcg(o1 + (size_t)j * D), O1);
      }
      store_out(h0, d0, O0);
      if (has1) store_out(h1, d1, O1);
    }
  } else {
    for (int i = threadIdx.x; i < g * D; i += blockDim.x) {
      const int h = i / D, d = i % D;
      const size_t pb = part + (size_t)h * nsplit;
      float M = -INFINITY;
#pragma unroll 8
      for (int j = 0; j < nsplit; ++j) M = fmaxf(M, __ldcg(ws_ml + (pb + j) * 2));
      float Lsum = 0.f, O = 0.f;
      if (M != -INFINITY) {
#pragma unroll 8
        for (int j = 0; j < nsplit; ++j) {
          const float mj = __ldcg(ws_ml + (pb + j) * 2);
          const float e = mj == -INFINITY ? 0.f : expf(mj - M);
          Lsum = fmaf(__ldcg(ws_ml + (pb + j) * 2 + 1), e, Lsum);
          O = fmaf(__ldcg(ws_o + (pb + j) * D + d), e, O);
        }
      }
      store_out(h, d, (valid && Lsum > 0.f) ? O / Lsum : 0.f);
    }
  }
  if (threadIdx.x == 0) ws_cnt[b * Hkv + kv] = 0u;  // ready for the next launch
  tl_exit(fz.tl);
}

}  // namespace qg
