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
#include <algorithm>
#include <mutex>

#include "attention_body.cuh"
#include "mma_sync.cuh"

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
      ws_cnt, fz, blockIdx.x, blockIdx.y, blockIdx.z, [&] {
        // the next kernel may be scheduled now: its own wait covers all of this one
        pdl_trigger();
        pdl_wait();
        tl_wait(fz.tl);
      });
}

// ---------------------------------------------------------------------------
// Cluster kernel (head_dim 32/64/128/256, at most 4 query heads per KV head).
//
// Grid (cs, Hkv, B) launched as clusters of cs CTAs along x: the cs CTAs of
// one (sequence, kv head) pair split its rows [0, L) into cs contiguous
// chunks of ch rows. Each row of K or V is D bf16 = D/8 lanes x 16 bytes, so
// one warp load instruction covers 32/(D/8) consecutive rows (a "slot");
// each lane keeps the 8 columns of its 16 bytes. A warp holds U slots of K
// and V in registers per batch, and two batches are in flight: the next one
// loads while the current one is scored (in the decode step the first two
// are issued before the programmatic-dependent-launch wait, since cached
// rows below the position are final). Per lane group (the lanes of one row):
// a running (max, sum, weighted V) per query head, updated once per batch.
// The warps' states merge in shared memory; the cluster's CTAs then merge in
// rank order through distributed shared memory (rank 0 reads every rank's
// partial), so the result is deterministic and needs no workspace, atomics
// or global round trip.
//
// Decode step (AttnFuse): every CTA norms and ropes its own query heads; the
// CTA whose chunk holds row p = position computes the new K and V rows, stores
// them in the cache for later steps and uses them from shared memory as row
// p, so no CTA reads a cache row this kernel writes.
// ---------------------------------------------------------------------------

namespace ac {

constexpr int kNW = 8;                 // warps per CTA
constexpr int kThreads = kNW * 32;
constexpr int kPortableCluster = 8;    // portable cluster size
constexpr int kMaxCluster = 16;        // non-portable, for long caches at few (sequence, kv head) pairs

template <int D>
struct Geo {
  static constexpr int LPR = D / 8;             // lanes per row (16 bytes each)
  static constexpr int RPI = 32 / LPR;          // rows per warp load instruction
  static constexpr int U = D >= 256 ? 2 : (D == 128 ? 3 : (RPI >= 8 ? 1 : 8 / RPI));  // slots per batch
  static constexpr int ROWS = kNW * U * RPI;    // rows per CTA batch
};

__device__ __forceinline__ uint4 ld_row16(const uint16_t* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ unsigned cluster_rank() {
  unsigned r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
               "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// fp32 at `p` (this CTA's shared memory) in the shared memory of CTA `rank`
// of the cluster.
__device__ __forceinline__ float ld_cluster(const float* p, unsigned rank) {
  const uint32_t local = (uint32_t)__cvta_generic_to_shared(p);
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

// fp32 v to the shared memory of CTA `rank` of the cluster, at the address
// `p` has in this CTA's shared memory.
__device__ __forceinline__ void st_cluster(float* p, float v, unsigned rank) {
  const uint32_t local = (uint32_t)__cvta_generic_to_shared(p);
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(rank));
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(remote), "f"(v) : "memory");
}

// Merge (m2, l2, o2) into (m, l, o): the larger max wins, the other side is
// scaled by exp(its max - new max). An empty side has max -inf, sum 0.
__device__ __forceinline__ void merge_state(float& m, float& l, float* o, float m2, float l2,
                                            const float* o2, int n) {
  const float M = fmaxf(m, m2);
  if (M == -INFINITY) return;
  const float a = expf(m - M), a2 = expf(m2 - M);
  l = l * a + l2 * a2;
  for (int i = 0; i < n; ++i) o[i] = o[i] * a + o2[i] * a2;
  m = M;
}

// One output element from the cluster's partials, merged in rank order:
// every rank's (max, sum, weighted value) is loaded first, so the reads of
// distributed shared memory overlap in one round trip, then combined. An
// empty rank has max -inf.
// MC: the largest cluster the instantiation serves (8, or 16 for the
// non-portable clusters of long caches; only those launches carry the wider
// merge).
template <int MC>
__device__ __forceinline__ float merge_cluster(const float* m, const float* l, const float* o,
                                               unsigned cs, bool valid) {
  float mv[MC], lv[MC], ov[MC];
#pragma unroll
  for (int j = 0; j < MC; ++j) {
    mv[j] = -INFINITY;
    lv[j] = ov[j] = 0.f;
    if (j < (int)cs) {
      mv[j] = ld_cluster(m, j);
      lv[j] = ld_cluster(l, j);
      ov[j] = ld_cluster(o, j);
    }
  }
  float M = -INFINITY;
#pragma unroll
  for (int j = 0; j < MC; ++j) M = fmaxf(M, mv[j]);
  float Ls = 0.f, O = 0.f;
  if (M != -INFINITY) {
#pragma unroll
    for (int j = 0; j < MC; ++j) {
      if (mv[j] == -INFINITY) continue;
      const float e = expf(mv[j] - M);
      Ls = fmaf(lv[j], e, Ls);
      O = fmaf(ov[j], e, O);
    }
  }
  return (valid && Ls > 0.f) ? O / Ls : 0.f;
}

// 4-byte cp.async granule helpers for the fused o_proj slice
__device__ __forceinline__ void cp_async_16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   (uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_8(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(
                   (uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src)
               : "memory");
}

template <int D, int GM, bool OPROJ, int MC = kPortableCluster>
__global__ void __launch_bounds__(kThreads, GM <= 2 ? 2 : 1)
attention_cluster_kernel(const float* q, const uint16_t* kc, const uint16_t* vc,
                         const int32_t* __restrict__ kv_len, const int32_t* __restrict__ pos_for_len,
                         void* out, int out_bf16, int H, int Hkv, int cap, float scale, int ch,
                         const AttnFuse fz) {
  using G = Geo<D>;
  constexpr int LPR = G::LPR, RPI = G::RPI, U = G::U;
  extern __shared__ __align__(16) uint8_t wslice[];  // fused o_proj: W_o rows of this CTA
  __shared__ float sq[GM][D];          // query heads (normed, roped) * scale
  __shared__ float kp[D], vp[D];       // the new row p (bf16 values), owner CTA only
  __shared__ float sp[GM];             // scores of row p
  __shared__ float wm[kNW][GM], wl[kNW][GM];
  __shared__ float wo[kNW][GM][D];
  __shared__ float cm[GM], cl[GM];     // this CTA's partial, read by rank 0
  __shared__ float co[GM][D];
  // kPush: every CTA stores its partial into rank 0's slots instead (one
  // cluster barrier, then rank 0 merges from its own shared memory) where
  // the slots fit a small static budget
  constexpr bool kPush = !OPROJ && MC * GM * (D + 2) * 4 <= 20480;
  __shared__ float pm[kPush ? MC : 1][GM], pl[kPush ? MC : 1][GM];
  __shared__ float po[kPush ? MC : 1][GM][D];

  tl_entry(fz.tl);
  attn_issue_prefetch(fz);
  const unsigned s = cluster_rank();
  const unsigned cs = gridDim.x;
  const int kv = blockIdx.y, b = blockIdx.z;
  const int g = H / Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = lane % LPR, r = lane / LPR;  // 16-byte chunk of the row; row in the slot
  const size_t head_base = ((size_t)b * Hkv + kv) * cap;
  const int t0 = (int)s * ch;

  // cached rows this CTA scores: [t0, tend)
  int tend = t0;
  bool valid = false;
  int p = -1;
  if (fz.on) {
    p = pos_for_len[b];
    valid = p >= 0 && p < cap;
    if (valid) tend = max(t0, min(t0 + ch, p));  // row p itself comes from shared memory
  }

  uint4 ka[U], va[U], kb[U], vb[U];
  auto load = [&](int batch, uint4(&kr)[U], uint4(&vr)[U]) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int t = t0 + ((batch * U + u) * kNW + warp) * RPI + r;
      if (t < tend) {
        const size_t off = (head_base + t) * D + c * 8;
        kr[u] = ld_row16(kc + off);
        vr[u] = ld_row16(vc + off);
      } else {
        kr[u] = vr[u] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
  };
  int nb = (tend - t0 + G::ROWS - 1) / G::ROWS;
  if (fz.on) {
    if (nb > 0) load(0, ka, va);
    if (nb > 1) load(1, kb, vb);
  }
  // fused o_proj: this CTA's W_o rows [s R, s R + R), the g*D columns of this
  // KV head's query heads, to shared memory (weights: no wait needed)
  const int gD = g * D;
  const int R = OPROJ ? fz.hidden / (int)cs : 0;
  // dynamic shared memory: W_o codes [R][gD], scales and biases [R][gD/64],
  // then ofin (rank 0: the head group's output, bf16 values) and xo (every
  // CTA's copy of it), gD floats each
  uint8_t* wcodes = wslice;
  uint16_t* wsc = reinterpret_cast<uint16_t*>(wslice + R * gD);
  uint16_t* wbi = wsc + R * (gD / 64);
  float* ofin = reinterpret_cast<float*>(wbi + R * (gD / 64));
  float* xo = ofin + gD;
  if constexpr (OPROJ) {
    const int HD = H * D, r0 = (int)s * R, c0 = kv * gD;
    const int chunks = R * gD / 16;
    for (int i = threadIdx.x; i < chunks; i += kThreads) {
      const int r = i / (gD / 16), c = (i % (gD / 16)) * 16;
      cp_async_16(wcodes + r * gD + c, fz.ow + (size_t)(r0 + r) * HD + c0 + c);
    }
    // gD / 64 bf16 scales and biases a row: gD / 64 * 2 bytes = 8 bytes for
    // gD = 256 (one granule), more granules for wider groups
    const int sbytes = gD / 64 * 2;
    for (int i = threadIdx.x; i < R * (sbytes / 8); i += kThreads) {
      const int r = i / (sbytes / 8), c = (i % (sbytes / 8)) * 4;
      const size_t gi = (size_t)(r0 + r) * (HD / 64) + c0 / 64 + c;
      cp_async_8(wsc + r * (gD / 64) + c, fz.os + gi);
      cp_async_8(wbi + r * (gD / 64) + c, fz.ob + gi);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  // the next kernel may be scheduled now: its own wait covers all of this one
  pdl_trigger();
  pdl_wait();
  tl_wait(fz.tl);
  if (!fz.on) {
    const int L = kv_len[b];
    valid = L >= 1 && L <= cap;
    tend = valid ? max(t0, min(t0 + ch, L)) : t0;
    nb = (tend - t0 + G::ROWS - 1) / G::ROWS;
    if (nb > 0) load(0, ka, va);
    if (nb > 1) load(1, kb, vb);
  }

  // ---- query heads (and, in the decode step, the new K/V row)
  const bool owner = fz.on && valid && p >= t0 && p < t0 + ch;
  if (!fz.on) {
    for (int i = threadIdx.x; i < g * D; i += kThreads)
      sq[i / D][i % D] = __ldcg(q + ((size_t)b * H + kv * g + i / D) * D + i % D) * scale;
  } else {
    const int tk = fz.tok[b];
    const bool write = owner && tk >= 0 && tk < fz.vocab;  // a bad token leaves the cache
    const float2* rcs = fz.rope + (size_t)b * (D / 2);
    const size_t row = (head_base + (valid ? p : 0)) * D;
    if (warp < g) {
      float* dst = sq[warp];
      norm_rope_head(q + ((size_t)b * H + kv * g + warp) * D, fz.qn, D, fz.eps, rcs, lane,
                     [&](int i, float v) { dst[i] = v * scale; });
    } else if (warp == g && owner) {
      norm_rope_head(fz.k + ((size_t)b * Hkv + kv) * D, fz.kn, D, fz.eps, rcs, lane,
                     [&](int i, float v) {
                       const uint16_t bits = f32_to_bf16_bits(v);
                       kp[i] = bf16_bits_to_f32(bits);
                       if (write) const_cast<uint16_t*>(kc)[row + i] = bits;
                     });
    } else if (warp == g + 1 && owner) {
      const float* vs = fz.v + ((size_t)b * Hkv + kv) * D;
      for (int d = lane; d < D; d += 32) {
        const uint16_t bits = f32_to_bf16_bits(__ldcg(vs + d));
        vp[d] = bf16_bits_to_f32(bits);
        if (write) const_cast<uint16_t*>(vc)[row + d] = bits;
      }
    }
  }
  __syncthreads();
  if (owner && warp < g) {  // score of row p for query head `warp`
    float d = 0.f;
    for (int i = lane; i < D; i += 32) d = fmaf(sq[warp][i], kp[i], d);
    d = warp_sum(d);
    if (lane == 0) sp[warp] = d;
  }

  // ---- this warp's rows: online softmax per lane group
  float qv[GM][8], o[GM][8], m[GM], l[GM];
#pragma unroll
  for (int h = 0; h < GM; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      qv[h][i] = h < g ? sq[h][c * 8 + i] : 0.f;
      o[h][i] = 0.f;
    }
  }
  auto process = [&](int batch, const uint4(&kr)[U], const uint4(&vr)[U]) {
    bool ok[U];
#pragma unroll
    for (int u = 0; u < U; ++u) ok[u] = t0 + ((batch * U + u) * kNW + warp) * RPI + r < tend;
#pragma unroll
    for (int h = 0; h < GM; ++h) {
      if (h >= g) break;
      float sc[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const uint4 k = kr[u];
        float d = qv[h][0] * bf16_lo(k.x);
        d = fmaf(qv[h][1], bf16_hi(k.x), d);
        d = fmaf(qv[h][2], bf16_lo(k.y), d);
        d = fmaf(qv[h][3], bf16_hi(k.y), d);
        d = fmaf(qv[h][4], bf16_lo(k.z), d);
        d = fmaf(qv[h][5], bf16_hi(k.z), d);
        d = fmaf(qv[h][6], bf16_lo(k.w), d);
        d = fmaf(qv[h][7], bf16_hi(k.w), d);
        sc[u] = d;
      }
#pragma unroll
      for (int off = LPR / 2; off >= 1; off >>= 1)
#pragma unroll
        for (int u = 0; u < U; ++u) sc[u] += __shfl_xor_sync(0xffffffffu, sc[u], off);
      float mx = m[h];
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (ok[u]) mx = fmaxf(mx, sc[u]);
      if (mx == -INFINITY) continue;
      const float a = expf(m[h] - mx);  // 0 while m is still -inf
      l[h] *= a;
#pragma unroll
      for (int i = 0; i < 8; ++i) o[h][i] *= a;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (!ok[u]) continue;
        const float pr = expf(sc[u] - mx);
        l[h] += pr;
        const uint4 v = vr[u];
        o[h][0] = fmaf(pr, bf16_lo(v.x), o[h][0]);
        o[h][1] = fmaf(pr, bf16_hi(v.x), o[h][1]);
        o[h][2] = fmaf(pr, bf16_lo(v.y), o[h][2]);
        o[h][3] = fmaf(pr, bf16_hi(v.y), o[h][3]);
        o[h][4] = fmaf(pr, bf16_lo(v.z), o[h][4]);
        o[h][5] = fmaf(pr, bf16_hi(v.z), o[h][5]);
        o[h][6] = fmaf(pr, bf16_lo(v.w), o[h][6]);
        o[h][7] = fmaf(pr, bf16_hi(v.w), o[h][7]);
      }
      m[h] = mx;
    }
  };
  for (int i = 0; i < nb; i += 2) {
    process(i, ka, va);
    if (i + 2 < nb) load(i + 2, ka, va);
    if (i + 1 < nb) {
      process(i + 1, kb, vb);
      if (i + 3 < nb) load(i + 3, kb, vb);
    }
  }

  // ---- merge the lane groups of the warp (lanes with the same chunk c)
#pragma unroll
  for (int off = LPR; off < 32; off <<= 1) {
#pragma unroll
    for (int h = 0; h < GM; ++h) {
      const float m2 = __shfl_xor_sync(0xffffffffu, m[h], off);
      const float l2 = __shfl_xor_sync(0xffffffffu, l[h], off);
      float o2[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) o2[i] = __shfl_xor_sync(0xffffffffu, o[h][i], off);
      merge_state(m[h], l[h], o[h], m2, l2, o2, 8);
    }
  }
  if (r == 0) {
#pragma unroll
    for (int h = 0; h < GM; ++h) {
      if (h >= g) break;
#pragma unroll
      for (int i = 0; i < 8; ++i) wo[warp][h][c * 8 + i] = o[h][i];
      if (c == 0) {
        wm[warp][h] = m[h];
        wl[warp][h] = l[h];
      }
    }
  }
  __syncthreads();

  // ---- this CTA's partial: its warps in order, then row p
  for (int i = threadIdx.x; i < g * D; i += kThreads) {
    const int h = i / D, d = i % D;
    float M = owner ? sp[h] : -INFINITY;
    for (int w = 0; w < kNW; ++w) M = fmaxf(M, wm[w][h]);
    float Ls = 0.f, O = 0.f;
    if (M != -INFINITY) {
      for (int w = 0; w < kNW; ++w) {
        const float e = wm[w][h] == -INFINITY ? 0.f : expf(wm[w][h] - M);
        Ls = fmaf(wl[w][h], e, Ls);
        O = fmaf(wo[w][h][d], e, O);
      }
      if (owner) {
        const float e = expf(sp[h] - M);
        Ls += e;
        O = fmaf(vp[d], e, O);
      }
    }
    if constexpr (kPush) {
      st_cluster(&po[s][h][d], O, 0);
      if (d == 0) {
        st_cluster(&pm[s][h], M, 0);
        st_cluster(&pl[s][h], Ls, 0);
      }
    } else {
      co[h][d] = O;
      if (d == 0) {
        cm[h] = M;
        cl[h] = Ls;
      }
    }
  }
  cluster_sync();  // every CTA's partial is in place (kPush: in rank 0's slots)

  if constexpr (kPush) {
    // ---- rank 0 merges its slots in rank order (the same arithmetic as
    // merge_cluster); the other CTAs are done
    if (s == 0) {
      for (int i = threadIdx.x; i < g * D; i += kThreads) {
        const int h = i / D, d = i % D;
        float M = -INFINITY;
        for (unsigned j = 0; j < cs; ++j) M = fmaxf(M, pm[j][h]);
        float Ls = 0.f, O = 0.f;
        if (M != -INFINITY) {
          for (unsigned j = 0; j < cs; ++j) {
            if (pm[j][h] == -INFINITY) continue;
            const float e = expf(pm[j][h] - M);
            Ls = fmaf(pl[j][h], e, Ls);
            O = fmaf(po[j][h][d], e, O);
          }
        }
        const float res = (valid && Ls > 0.f) ? O / Ls : 0.f;
        const size_t oi = ((size_t)b * H + kv * g + h) * D + d;
        if (out_bf16)
          reinterpret_cast<uint16_t*>(out)[oi] = f32_to_bf16_bits(res);
        else
          reinterpret_cast<float*>(out)[oi] = res;
      }
    }
    tl_exit(fz.tl);
    return;
  }

  // ---- rank 0 merges the cluster's partials in rank order
  if (s == 0) {
    for (int i = threadIdx.x; i < g * D; i += kThreads) {
      const int h = i / D, d = i % D;
      const float res = merge_cluster<MC>(&cm[h], &cl[h], &co[h][d], cs, valid);
      const size_t oi = ((size_t)b * H + kv * g + h) * D + d;
      if (out_bf16)
        reinterpret_cast<uint16_t*>(out)[oi] = f32_to_bf16_bits(res);
      else
        reinterpret_cast<float*>(out)[oi] = res;
      if constexpr (OPROJ) ofin[i] = bf16_bits_to_f32(f32_to_bf16_bits(res));
    }
  }
  cluster_sync();  // no CTA leaves while rank 0 still reads its shared memory
  if constexpr (OPROJ) {
    // the head group's bf16 output from rank 0, then the o_proj partial rows
    for (int i = threadIdx.x; i < gD; i += kThreads) xo[i] = ld_cluster(&ofin[i], 0);
    cluster_sync();  // rank 0 stays until every CTA has read its output
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
    // thread t: row t / tpr of the slice, columns [p * cpt, (p + 1) * cpt)
    // (whole 64-column groups) with p = t % tpr; per group s * sum(q x) +
    // beta * sum(x), products exact in fp32; the tpr parts then meet by
    // shuffles in a fixed order
    const int tpr = kThreads / R, cpt = gD / tpr;
    const int r = threadIdx.x / tpr, p = threadIdx.x % tpr;
    float acc = 0.f;
    for (int c0 = p * cpt; c0 < (p + 1) * cpt; c0 += 64) {
      const uint32_t* qw = reinterpret_cast<const uint32_t*>(wcodes + r * gD + c0);
      float sq = 0.f, sx = 0.f;
#pragma unroll 4
      for (int j = 0; j < 16; ++j) {
        const uint32_t w = qw[j];
        const float* xv = xo + c0 + 4 * j;
        sq = fmaf(byte_to_f32<0>(w), xv[0], sq);
        sq = fmaf(byte_to_f32<1>(w), xv[1], sq);
        sq = fmaf(byte_to_f32<2>(w), xv[2], sq);
        sq = fmaf(byte_to_f32<3>(w), xv[3], sq);
        sx += (xv[0] + xv[1]) + (xv[2] + xv[3]);
      }
      const int gi = r * (gD / 64) + c0 / 64;
      acc = fmaf(bf16_bits_to_f32(wsc[gi]), sq, fmaf(bf16_bits_to_f32(wbi[gi]), sx, acc));
    }
    for (int off = 1; off < tpr; off <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (p == 0)
      fz.opart[((size_t)b * Hkv + kv) * fz.hidden + (size_t)s * R + r] = valid ? acc : __int_as_float(0x7fc00000);
  }
  tl_exit(fz.tl);
}

// ---------------------------------------------------------------------------
// Tensor-core kernel for long caches and many sequences (head_dim 64 or 128,
// at most 8 query heads per KV head).
//
// Same grid, clusters, row chunks, decode-step fusion and rank-order cluster
// merge as the cluster kernel above; what changes is how a CTA scores its
// rows. Blocks of 64 cached rows of K and V are staged in shared memory by
// cp.async, three blocks in flight, 16-byte chunks XOR-swizzled by row so
// that ldmatrix reads are conflict-free. Each of the 4 warps takes 16 rows
// of a block: S = Q K^T and O += P V run on the tensor cores (mma.sync
// m16n8k16, bf16 operands, fp32 accumulation) with the g query heads as the
// A operand's first g rows. The fp32 query (normed, roped, times the scale)
// and the fp32 softmax weights enter as bf16 pairs hi + lo with
// hi = bf16(x), lo = bf16(x - hi), so |x - hi - lo| <= 2^-16 |x| and the
// products keep fp32-grade accuracy; the online softmax (max, sum) is in fp32
// per query head over the quad of lanes that holds its row.
// ---------------------------------------------------------------------------

constexpr int kMW = 4;                 // warps per CTA
constexpr int kMThreads = kMW * 32;
constexpr int kMB = 64;                // cached rows per staged block
constexpr int kMStages = 3;            // blocks in flight
constexpr int kMG = 8;                 // query heads per KV head, at most

template <int D>
constexpr int mma_smem_bytes() {
  return kMStages * 2 * kMB * D * 2;   // [stage][K, V][kMB][D] bf16
}

template <int D>
__global__ void __launch_bounds__(kMThreads, 2)
attention_mma_kernel(const float* q, const uint16_t* kc, const uint16_t* vc,
                     const int32_t* __restrict__ kv_len, const int32_t* __restrict__ pos_for_len,
                     void* out, int out_bf16, int H, int Hkv, int cap, float scale, int ch,
                     const AttnFuse fz) {
  using namespace mm;
  constexpr int KS = D / 16;           // k-steps of Q K^T
  constexpr int CPR = D / 8;           // 16-byte chunks per row
  constexpr int TILE = kMB * D * 2;    // bytes of one K or V block
  extern __shared__ __align__(128) uint8_t stage[];
  __shared__ float sq[kMG][D];         // query heads (normed, roped) * scale
  __shared__ float kp[D], vp[D];       // the new row p (bf16 values), owner CTA only
  __shared__ float sp[kMG];            // scores of row p
  __shared__ float wm[kMW][kMG], wl[kMW][kMG];
  __shared__ float cm[kMG], cl[kMG];   // this CTA's partial, read by rank 0
  __shared__ float co[kMG][D];

  tl_entry(fz.tl);
  attn_issue_prefetch(fz);
  const unsigned s = cluster_rank();
  const unsigned cs = gridDim.x;
  const int kv = blockIdx.y, b = blockIdx.z;
  const int g = H / Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const size_t head_base = ((size_t)b * Hkv + kv) * cap;
  const int t0 = (int)s * ch;

  // cached rows this CTA scores: [t0, tend)
  int tend = t0;
  bool valid = false;
  int p = -1;
  if (fz.on) {
    p = pos_for_len[b];
    valid = p >= 0 && p < cap;
    if (valid) tend = max(t0, min(t0 + ch, p));  // row p itself comes from shared memory
  }
  const uint32_t sbase = smem_u32(stage);
  // block j of the chunk into stage buffer j % kMStages; rows at or past
  // tend are zero-filled (their scores are masked to -inf)
  auto load_block = [&](int j) {
    const int tb = t0 + j * kMB;
    const uint32_t kd = sbase + (uint32_t)((j % kMStages) * 2 * TILE);
    const uint32_t vd = kd + TILE;
#pragma unroll
    for (int i = 0; i < kMB * CPR / kMThreads; ++i) {
      const int idx = tid + i * kMThreads;
      const int row = idx / CPR, c = idx % CPR;
      const int t = tb + row;
      const bool ok = t < tend;
      const size_t off = (head_base + (ok ? t : 0)) * D + c * 8;
      const uint32_t so = swz<D>(row, c * 8);
      cp_async16(kd + so, kc + off, ok);
      cp_async16(vd + so, vc + off, ok);
    }
  };
  int nb = (tend - t0 + kMB - 1) / kMB;
  auto prologue = [&] {
#pragma unroll
    for (int j = 0; j < kMStages - 1; ++j) {
      if (j < nb) load_block(j);
      cp_async_commit();
    }
  };
  // decode step: the cached rows below the position are final, so the first
  // blocks are in flight before the programmatic-dependent-launch wait
  if (fz.on) prologue();
  pdl_trigger();
  pdl_wait();
  tl_wait(fz.tl);
  if (!fz.on) {
    const int L = kv_len[b];
    valid = L >= 1 && L <= cap;
    tend = valid ? max(t0, min(t0 + ch, L)) : t0;
    nb = (tend - t0 + kMB - 1) / kMB;
    prologue();
  }

  // ---- query heads (and, in the decode step, the new K/V row)
  const bool owner = fz.on && valid && p >= t0 && p < t0 + ch;
  if (!fz.on) {
    for (int i = tid; i < g * D; i += kMThreads)
      sq[i / D][i % D] = __ldcg(q + ((size_t)b * H + kv * g + i / D) * D + i % D) * scale;
  } else {
    const int tk = fz.tok[b];
    const bool write = owner && tk >= 0 && tk < fz.vocab;  // a bad token leaves the cache
    const float2* rcs = fz.rope + (size_t)b * (D / 2);
    const size_t row = (head_base + (valid ? p : 0)) * D;
    // items 0..g-1: query heads; g: the new K row; g + 1: the new V row
    for (int it = warp; it < g + 2; it += kMW) {
      if (it < g) {
        float* dst = sq[it];
        norm_rope_head(q + ((size_t)b * H + kv * g + it) * D, fz.qn, D, fz.eps, rcs, lane,
                       [&](int i, float v) { dst[i] = v * scale; });
      } else if (it == g && owner) {
        norm_rope_head(fz.k + ((size_t)b * Hkv + kv) * D, fz.kn, D, fz.eps, rcs, lane,
                       [&](int i, float v) {
                         const uint16_t bits = f32_to_bf16_bits(v);
                         kp[i] = bf16_bits_to_f32(bits);
                         if (write) const_cast<uint16_t*>(kc)[row + i] = bits;
                       });
      } else if (it == g + 1 && owner) {
        const float* vs = fz.v + ((size_t)b * Hkv + kv) * D;
        for (int d = lane; d < D; d += 32) {
          const uint16_t bits = f32_to_bf16_bits(__ldcg(vs + d));
          vp[d] = bf16_bits_to_f32(bits);
          if (write) const_cast<uint16_t*>(vc)[row + d] = bits;
        }
      }
    }
  }
  __syncthreads();
  if (owner) {  // score of row p for each query head
    for (int h = warp; h < g; h += kMW) {
      float d = 0.f;
      for (int i = lane; i < D; i += 32) d = fmaf(sq[h][i], kp[i], d);
      d = warp_sum(d);
      if (lane == 0) sp[h] = d;
    }
  }

  // ---- A fragments of Q: row qr = lane / 4 (a query head when qr < g; rows
  // 8..15 of the m16 tile are zero), columns 16 ks + 2 (lane % 4) + {0, 1}
  // and + 8, as hi and lo bf16 pairs
  const int qr = lane >> 2, qc = (lane & 3) * 2;
  uint32_t qhi[KS][2], qlo[KS][2];
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int d = ks * 16 + hf * 8 + qc;
      const float x0 = qr < g ? sq[qr][d] : 0.f, x1 = qr < g ? sq[qr][d + 1] : 0.f;
      const float h0 = bf16r(x0), h1 = bf16r(x1);
      qhi[ks][hf] = pack_bf16(h0, h1);
      qlo[ks][hf] = pack_bf16(x0 - h0, x1 - h1);
    }
  }

  // ---- this warp's 16 rows of each block: online softmax of query head qr
  float o[D / 8][4];
#pragma unroll
  for (int j = 0; j < D / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;  // l_run: this lane's share of the sum
  for (int j = 0; j < nb; ++j) {
    cp_async_wait<kMStages - 2>();
    __syncthreads();  // block j landed for every thread; buffer (j - 1) % kMStages is free
    if (j + kMStages - 1 < nb) load_block(j + kMStages - 1);
    cp_async_commit();
    const uint32_t kb = sbase + (uint32_t)((j % kMStages) * 2 * TILE);
    const uint32_t vb = kb + TILE;

    // S = Q K^T over rows warp*16 + [0, 16): n-tiles of 8 rows; ldmatrix
    // (no transpose) of K rows gives the col-major B fragment directly
    float sacc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ks += 2) {
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const int row = warp * 16 + nt * 8 + (lane & 7);
        uint32_t r0, r1, r2, r3;
        ldsm_x4(kb + swz<D>(row, (ks * 2 + (lane >> 3)) * 8), r0, r1, r2, r3);
        mma_bf16(sacc[nt], qhi[ks][0], 0u, qhi[ks][1], 0u, r0, r1);
        mma_bf16(sacc[nt], qlo[ks][0], 0u, qlo[ks][1], 0u, r0, r1);
        mma_bf16(sacc[nt], qhi[ks + 1][0], 0u, qhi[ks + 1][1], 0u, r2, r3);
        mma_bf16(sacc[nt], qlo[ks + 1][0], 0u, qlo[ks + 1][1], 0u, r2, r3);
      }
    }
    // this lane's scores: rows t0 + j*kMB + warp*16 + nt*8 + qc + {0, 1}
    const int tb = t0 + j * kMB + warp * 16 + qc;
    float sv[4];
    float mx = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float v = tb + nt * 8 + e < tend ? sacc[nt][e] : -INFINITY;
        sv[nt * 2 + e] = v;
        mx = fmaxf(mx, v);
      }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float mnew = fmaxf(m_run, mx);
    float pr[4] = {0.f, 0.f, 0.f, 0.f};
    if (mnew != -INFINITY) {
      const float a = expf(m_run - mnew);  // 0 while m_run is still -inf
      l_run *= a;
#pragma unroll
      for (int dn = 0; dn < D / 8; ++dn) {
        o[dn][0] *= a;
        o[dn][1] *= a;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) pr[i] = expf(sv[i] - mnew);  // masked rows: 0
      l_run += (pr[0] + pr[1]) + (pr[2] + pr[3]);
      m_run = mnew;
    }
    // O += P V: P's A fragment is the score layout (columns qc + {0,1} of
    // n-tile 0, then of n-tile 1); ldmatrix.trans of V rows gives the B
    // fragment (k = row, n = column of the head)
    const float h0 = bf16r(pr[0]), h1 = bf16r(pr[1]), h2 = bf16r(pr[2]), h3 = bf16r(pr[3]);
    const uint32_t pa_h = pack_bf16(h0, h1), pb_h = pack_bf16(h2, h3);
    const uint32_t pa_l = pack_bf16(pr[0] - h0, pr[1] - h1), pb_l = pack_bf16(pr[2] - h2, pr[3] - h3);
#pragma unroll
    for (int dn = 0; dn < D / 8; dn += 2) {
      const int row = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
      uint32_t r0, r1, r2, r3;
      ldsm_x4_t(vb + swz<D>(row, (dn + (lane >> 4)) * 8), r0, r1, r2, r3);
      mma_bf16(o[dn], pa_h, 0u, pb_h, 0u, r0, r1);
      mma_bf16(o[dn], pa_l, 0u, pb_l, 0u, r0, r1);
      mma_bf16(o[dn + 1], pa_h, 0u, pb_h, 0u, r2, r3);
      mma_bf16(o[dn + 1], pa_l, 0u, pb_l, 0u, r2, r3);
    }
  }
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);

  // ---- the warps' states to shared memory; wo [kMW][kMG][D] reuses the
  // staging buffers once every copy has landed and every warp is done
  cp_async_wait<0>();
  __syncthreads();
  float* wo = reinterpret_cast<float*>(stage);
  if (qr < g) {
#pragma unroll
    for (int dn = 0; dn < D / 8; ++dn) {
      wo[(warp * kMG + qr) * D + dn * 8 + qc] = o[dn][0];
      wo[(warp * kMG + qr) * D + dn * 8 + qc + 1] = o[dn][1];
    }
    if ((lane & 3) == 0) {
      wm[warp][qr] = m_run;
      wl[warp][qr] = l_run;
    }
  }
  __syncthreads();

  // ---- this CTA's partial: its warps in order, then row p
  for (int i = tid; i < g * D; i += kMThreads) {
    const int h = i / D, d = i % D;
    float M = owner ? sp[h] : -INFINITY;
    for (int w = 0; w < kMW; ++w) M = fmaxf(M, wm[w][h]);
    float Ls = 0.f, O = 0.f;
    if (M != -INFINITY) {
      for (int w = 0; w < kMW; ++w) {
        const float e = wm[w][h] == -INFINITY ? 0.f : expf(wm[w][h] - M);
        Ls = fmaf(wl[w][h], e, Ls);
        O = fmaf(wo[(w * kMG + h) * D + d], e, O);
      }
      if (owner) {
        const float e = expf(sp[h] - M);
        Ls += e;
        O = fmaf(vp[d], e, O);
      }
    }
    co[h][d] = O;
    if (d == 0) {
      cm[h] = M;
      cl[h] = Ls;
    }
  }
  cluster_sync();  // every CTA's partial is in its shared memory

  // ---- rank 0 merges the cluster's partials in rank order
  if (s == 0) {
    for (int i = tid; i < g * D; i += kMThreads) {
      const int h = i / D, d = i % D;
      const float res = merge_cluster<kPortableCluster>(&cm[h], &cl[h], &co[h][d], cs, valid);
      const size_t oi = ((size_t)b * H + kv * g + h) * D + d;
      if (out_bf16)
        reinterpret_cast<uint16_t*>(out)[oi] = f32_to_bf16_bits(res);
      else
        reinterpret_cast<float*>(out)[oi] = res;
    }
  }
  cluster_sync();  // no CTA leaves while rank 0 still reads its shared memory
  tl_exit(fz.tl);
}

// Whether the tensor-core kernel takes the shape: head_dim 64 or 128, at
// most 8 query heads per KV head, and at least 2^16 cached rows over all
// (sequence, kv head) pairs (below that the cluster kernel's lighter
// prologue wins).
constexpr long long kMmaMinRows = 1LL << 16;
inline bool mma_ok(int B, int H, int Hkv, int D, int cap) {
  if (!(D == 64 || D == 128) || Hkv < 1 || H % Hkv != 0) return false;
  const int g = H / Hkv;
  if (g < 1 || g > kMG) return false;
  return (long long)B * Hkv * cap >= kMmaMinRows;
}

// CTAs per (sequence, kv head) for the tensor-core kernel: as many as fit
// in one wave of two CTAs per SM (at most 8, a portable cluster), each a
// whole number of 64-row blocks; `ch` = rows per CTA.
inline void mma_plan(int B, int Hkv, int cap, int& cs, int& ch) {
  const long long pairs = (long long)B * Hkv;
  long long c = (2LL * num_sms()) / pairs;
  c = std::max<long long>(1, std::min<long long>(c, kPortableCluster));
  const int blocks = (cap + kMB - 1) / kMB;
  c = std::min<long long>(c, blocks);
  ch = (int)((blocks + c - 1) / c) * kMB;
  cs = (cap + ch - 1) / ch;
}

template <int D>
cudaError_t launch_mma(const float* q, const uint16_t* kc, const uint16_t* vc,
                       const int32_t* kv_len, const int32_t* pos_for_len, void* out,
                       bool out_bf16, int B, int H, int Hkv, int cap, float scale,
                       cudaStream_t st, bool pdl, const AttnFuse& fz) {
  int cs = 1, ch = cap;
  mma_plan(B, Hkv, cap, cs, ch);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cs, Hkv, B);
  cfg.blockDim = dim3(kMThreads);
  cfg.dynamicSmemBytes = mma_smem_bytes<D>();
  ensure_smem((const void*)attention_mma_kernel<D>, (int)cfg.dynamicSmemBytes);
  cfg.stream = st;
  cudaLaunchAttribute a[2];
  a[0].id = cudaLaunchAttributeClusterDimension;
  a[0].val.clusterDim.x = cs;
  a[0].val.clusterDim.y = 1;
  a[0].val.clusterDim.z = 1;
  a[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = a;
  cfg.numAttrs = pdl ? 2 : 1;
  count_launch();
  return cudaLaunchKernelEx(&cfg, attention_mma_kernel<D>, q, kc, vc, kv_len, pos_for_len, out,
                            (int)out_bf16, H, Hkv, cap, scale, ch, fz);
}

// Whether the cluster kernel takes the shape.
inline bool cluster_ok(int H, int Hkv, int D) {
  const int g = H / Hkv;
  return (D == 32 || D == 64 || D == 128 || D == 256) && g >= 1 && g <= 4 && H % Hkv == 0;
}

// CTAs per (sequence, kv head): enough CTAs for about four waves of two
// CTAs per SM, chunks of at least 16 rows, and at most 8 (a portable
// cluster) unless the chunks stay at least 128 rows long, up to 16. Measured
// on the B200: clusters of 16 made the 0.6B step (KV 512, 32-row chunks)
// slower, while a batch-1 cache of 2048 rows leaves 8 kv heads x 8 CTAs =
// 64 CTAs, each with 256 rows to score.
inline int cluster_size(int B, int Hkv, int cap) {
  const long long pairs = (long long)B * Hkv;
  long long cs = (8LL * num_sms() + pairs - 1) / pairs;
  cs = std::min<long long>(cs, (cap + 15) / 16);
  const long long most = std::max<long long>(kPortableCluster, std::min<long long>(kMaxCluster, cap / 128));
  cs = std::max<long long>(1, std::min<long long>(cs, most));
  return (int)cs;
}

// Whether the fused o_proj takes the launch: rows hidden / cs per CTA, each
// thread whole 64-column groups of the head group's g*D columns, and the
// slice within a dynamic shared-memory budget.
inline int oproj_smem(int hidden, int cs, int gD) {
  const int R = hidden / cs;
  return R * gD + 2 * R * (gD / 64) * 2 + 2 * gD * 4;
}
inline bool oproj_ok(int hidden, int cs, int gD) {
  if (cs < 1 || hidden % cs != 0) return false;
  const int R = hidden / cs;
  if (R < 1 || R > kThreads || kThreads % R != 0) return false;
  const int tpr = kThreads / R;
  if (gD % 64 != 0 || gD % tpr != 0 || (gD / tpr) % 64 != 0 || (gD / 64 * 2) % 8 != 0)
    return false;
  if (tpr > 32) return false;
  return oproj_smem(hidden, cs, gD) <= 96 * 1024;
}

template <int D, int GM, bool OPROJ>
cudaError_t launch(const float* q, const uint16_t* kc, const uint16_t* vc, const int32_t* kv_len,
                   const int32_t* pos_for_len, void* out, bool out_bf16, int B, int H, int Hkv,
                   int cap, float scale, cudaStream_t st, bool pdl, const AttnFuse& fz) {
  const int cs = cluster_size(B, Hkv, cap);
  const int ch = (cap + cs - 1) / cs;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cs, Hkv, B);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = OPROJ ? oproj_smem(fz.hidden, cs, (H / Hkv) * D) : 0;
  if (OPROJ)
    ensure_smem((const void*)attention_cluster_kernel<D, GM, true>, (int)cfg.dynamicSmemBytes);
  const bool wide = !OPROJ && cs > kPortableCluster;  // (the fused o_proj keeps portable clusters)
  if (wide) {
    static std::once_flag once;
    std::call_once(once, [] {
      cudaFuncSetAttribute((const void*)attention_cluster_kernel<D, GM, false, kMaxCluster>,
                           cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    });
  }
  cfg.stream = st;
  cudaLaunchAttribute a[2];
  a[0].id = cudaLaunchAttributeClusterDimension;
  a[0].val.clusterDim.x = cs;
  a[0].val.clusterDim.y = 1;
  a[0].val.clusterDim.z = 1;
  a[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = a;
  cfg.numAttrs = pdl ? 2 : 1;
  count_launch();
  if (wide)
    return cudaLaunchKernelEx(&cfg, attention_cluster_kernel<D, GM, false, kMaxCluster>, q, kc, vc,
                              kv_len, pos_for_len, out, (int)out_bf16, H, Hkv, cap, scale, ch, fz);
  return cudaLaunchKernelEx(&cfg, attention_cluster_kernel<D, GM, OPROJ>, q, kc, vc, kv_len,
                            pos_for_len, out, (int)out_bf16, H, Hkv, cap, scale, ch, fz);
}

template <int D>
cudaError_t launch_d(const float* q, const uint16_t* kc, const uint16_t* vc, const int32_t* kv_len,
                     const int32_t* pos_for_len, void* out, bool out_bf16, int B, int H, int Hkv,
                     int cap, float scale, cudaStream_t st, bool pdl, const AttnFuse& fz) {
  const int g = H / Hkv;
  if (fz.ow) {  // the caller checked oproj_ok
    if (g <= 1)
      return launch<D, 1, true>(q, kc, vc, kv_len, pos_for_len, out, out_bf16, B, H, Hkv, cap,
                                scale, st, pdl, fz);
    if (g <= 2)
      return launch<D, 2, true>(q, kc, vc, kv_len, pos_for_len, out, out_bf16, B, H, Hkv, cap,
                                scale, st, pdl, fz);
    return launch<D, 4, true>(q, kc, vc, kv_len, pos_for_len, out, out_bf16, B, H, Hkv, cap,
                              scale, st, pdl, fz);
  }
  if (g <= 1)
    return launch<D, 1, false>(q, kc, vc, kv_len, pos_for_len, out, out_bf16, B, H, Hkv, cap,
                               scale, st, pdl, fz);
  if (g <= 2)
    return launch<D, 2, false>(q, kc, vc, kv_len, pos_for_len, out, out_bf16, B, H, Hkv, cap,
                               scale, st, pdl, fz);
  return launch<D, 4, false>(q, kc, vc, kv_len, pos_for_len, out, out_bf16, B, H, Hkv, cap, scale,
                             st, pdl, fz);
}

}  // namespace ac

static cudaError_t attention_launch_any(const float* q, const uint16_t* kc, const uint16_t* vc,
                                        const int32_t* kv_len, const int32_t* pos_for_len,
                                        void* out, bool out_bf16, int B, int H, int Hkv, int D,
                                        int cap, float scale, void* ws, cudaStream_t st, bool pdl,
                                        const AttnFuse& fz) {
  if (!fz.ow && ac::mma_ok(B, H, Hkv, D, cap)) {
    if (D == 64)
      return ac::launch_mma<64>(q, kc, vc, kv_len, pos_for_len, out, out_bf16, B, H, Hkv, cap,
                                scale, st, pdl, fz);
    return ac::launch_mma<128>(q, kc, vc, kv_len, pos_for_len, out, out_bf16, B, H, Hkv, cap,
                               scale, st, pdl, fz);
  }
  if (ac::cluster_ok(H, Hkv, D)) {
    switch (D) {
      case 32:
        return ac::launch_d<32>(q, kc, vc, kv_len, pos_for_len, out, out_bf16, B, H, Hkv, cap,
                                scale, st, pdl, fz);
      case 64:
        return ac::launch_d<64>(q, kc, vc, kv_len, pos_for_len, out, out_bf16, B, H, Hkv, cap,
                                scale, st, pdl, fz);
      case 128:
        return ac::launch_d<128>(q, kc, vc, kv_len, pos_for_len, out, out_bf16, B, H, Hkv, cap,
                                 scale, st, pdl, fz);
      default:
        return ac::launch_d<256>(q, kc, vc, kv_len, pos_for_len, out, out_bf16, B, H, Hkv, cap,
                                 scale, st, pdl, fz);
    }
  }
  // other head sizes and groups: the split kernel with a workspace merge
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
                                  cudaStream_t st, bool pdl, const Prefetch* pf,
                                  const OProjFuse* op) {
  AttnFuse fz = {};
  if (op) {
    fz.ow = reinterpret_cast<const uint8_t*>(op->w);
    fz.os = op->s;
    fz.ob = op->b;
    fz.opart = op->part;
    fz.hidden = op->hidden;
  }
  fz.on = 1;
  fz.k = k;
  fz.v = v;
  fz.qn = q_norm;
  fz.kn = k_norm;
  fz.tok = tokens;
  fz.vocab = vocab;
  fz.eps = eps;
  fz.rope = rope;
  if (pf) fz.pf = *pf;
  fz.tl = tl_take(0);
  return attention_launch_any(q, kc, vc, nullptr, positions, out, true, B, H, Hkv, D, cap, scale,
                              ws, st, pdl, fz);
}

bool attention_oproj_fusable(int B, int H, int Hkv, int D, int cap, int hidden) {
  if (!ac::cluster_ok(H, Hkv, D) || ac::mma_ok(B, H, Hkv, D, cap)) return false;
  const int cs = ac::cluster_size(B, Hkv, cap);
  // (the fused o_proj is built for portable clusters only)
  return cs <= ac::kPortableCluster && ac::oproj_ok(hidden, cs, (H / Hkv) * D);
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
  // Only the split kernel touches scratch; the cluster and tensor-core
  // kernels merge through distributed shared memory, so their shapes are not
  // limited by the array.
  const bool split = !ac::cluster_ok(H, Hkv, D) && !ac::mma_ok(B, H, Hkv, D, cap);
  if (split) {
    const size_t need = attention_ws_bytes(B, H, Hkv, D, cap);
    QG_REQUIRE(need <= kAttnStaticScratchBytes, QG_ERR_WORKSPACE_TOO_SMALL,
               "qg_decode_attention_static_scratch: this shape needs %zu bytes of scratch, more "
               "than the fixed %zu; use qg_decode_attention with a caller workspace",
               need, kAttnStaticScratchBytes);
  }
  void* ws = nullptr;
  cudaError_t e = attn_scratch_address(&ws);
  if (e != cudaSuccess) {
    set_error("qg_decode_attention_static_scratch: scratch address lookup failed: %s",
              cudaGetErrorString(e));
    return QG_ERR_CUDA;
  }
  cudaStream_t s = (cudaStream_t)stream;
  if (split) {
    // the ticket counters must start at zero (the kernel also leaves them at
    // zero; a cleared start does not depend on how the last call ended)
    const size_t off = attention_ws_counter_offset(B, H, Hkv, D, cap);
    e = cudaMemsetAsync(reinterpret_cast<uint8_t*>(ws) + off, 0,
                        (size_t)B * Hkv * sizeof(unsigned int), s);
    if (e != cudaSuccess) {
      set_error("qg_decode_attention_static_scratch: %s", cudaGetErrorString(e));
      return QG_ERR_CUDA;
    }
  }
  attention_launch(q, k_cache, v_cache, kv_len, nullptr, out, out_dtype == QG_BF16, B, H, Hkv, D,
                   cap, scale, ws, s, false);
  return check_launch("qg_decode_attention_static_scratch");
}
