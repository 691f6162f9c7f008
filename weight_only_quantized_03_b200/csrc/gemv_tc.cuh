// Tensor-core affine-INT8 GEMV: the per-CTA body of the kernel in
// gemv_affine8_tc.cu (which describes the design).
#pragma once

#include "qg_internal.cuh"

namespace qg {
namespace gtc {

// Warps per CTA (template W): 16 with one batch tile for streaming matrices
// (128 registers a thread, the whole register file: the most loads in
// flight); 8 for decode-layer matrices (one batch tile, about 234 registers)
// and with two batch tiles (about 255).
constexpr int kRB = 16;        // rows per block (mma M)
constexpr int kSC = 512;       // columns per super-chunk
constexpr int kMaxSegs = 4;
constexpr int kMaxB = 8;       // batch rows per CTA: two n-tiles of four
constexpr int kMaxBatch = 32;  // batch rows per launch: tiles of kMaxB along gridDim.y

struct Seg {
  const uint8_t* w;
  const uint16_t* s;
  const uint16_t* b;
  void* y;
  const float* res;
  int N;
  int y_bf16;
  int blk0;  // first global block index of this segment
};

// How the GEMV input is formed in the prologue (every CTA forms all of it):
//   kXBf16     x bf16 [B][K] as given;
//   kXRmsNorm  bf16(xa / sqrt(mean(xa^2) + eps) * nw) per batch row, xa fp32;
//   kXSiluMul  bf16(silu(xa) * xb), xa = gate and xb = up, both fp32.
//   kXRmsNormParts  as kXRmsNorm of xa + sum_{j < nparts} parts[j] (the
//                   o_proj partial rows of the fused attention, summed in
//                   order j = 0, 1, ...); CTA 0 also stores that sum (the
//                   residual stream after o_proj) to xsum.
enum XMode { kXBf16 = 0, kXRmsNorm = 1, kXSiluMul = 2, kXRmsNormParts = 3 };

struct Params {
  Seg seg[kMaxSegs];
  int nseg, K, B, nblocks, S, xmode;
  const uint16_t* x;   // kXBf16
  const float* xa;     // kXRmsNorm, kXSiluMul
  const float* xb;     // kXSiluMul
  const uint16_t* nw;  // kXRmsNorm weight, bf16 [K]
  float eps;
  uint16_t* xout;      // optional: CTA 0 records the formed bf16 input [B][K]
  const float* parts;  // kXRmsNormParts: [B][nparts][K]
  int nparts;
  float* xsum;         // kXRmsNormParts: CTA 0 stores xa + sum(parts) [B][K]
  Prefetch pf;         // L2 prefetch work for a later kernel (pf.n == 0, pf.kv.kc null: none)
  TlRec* tl;           // timeline record of this launch, or null
};

__device__ __forceinline__ void ld_w8(const uint8_t* p, uint64_t pol, uint32_t* r) {
  asm volatile(
      "ld.global.nc.L1::no_allocate.L2::cache_hint.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8], %9;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7])
      : "l"(p), "l"(pol));
}
__device__ __forceinline__ uint32_t ld_u32_nc(const uint16_t* p) {
  uint32_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ void mma_f16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// which segment a global block index belongs to
__device__ __forceinline__ int seg_of(const Params& P, int blk) {
  int si = 0;
#pragma unroll
  for (int i = 1; i < kMaxSegs; ++i)
    if (i < P.nseg && blk >= P.seg[i].blk0) si = i;
  return si;
}

// Per-lane pointers into one 16-row block: rows g and g + 8 (clamped to the
// matrix; rows past N are loaded but never stored). dr = row distance.
struct Rows {
  const uint8_t* w;
  const uint16_t* s;
  const uint16_t* b;
  int dr;
};

__device__ __forceinline__ Rows rows_of(const Params& P, int blk, int g, int t) {
  const Seg& S = P.seg[seg_of(P, blk)];
  const int row0 = (blk - S.blk0) * kRB;
  const int r0 = min(row0 + g, S.N - 1), r1 = min(row0 + g + 8, S.N - 1);
  const int K = P.K, Kg = K / 64;
  Rows R;
  R.w = S.w + (size_t)r0 * K + 32 * t;
  R.s = S.s + (size_t)r0 * Kg + 2 * t;
  R.b = S.b + (size_t)r0 * Kg + 2 * t;
  R.dr = r1 - r0;
  return R;
}

__device__ __forceinline__ void load_scales(const Rows& R, int Kg, int sc, uint32_t (&v)[4]) {
  const int o1 = R.dr * Kg + sc * 8;
  v[0] = ld_u32_nc(R.s + sc * 8);
  v[1] = ld_u32_nc(R.s + o1);
  v[2] = ld_u32_nc(R.b + sc * 8);
  v[3] = ld_u32_nc(R.b + o1);
}
__device__ __forceinline__ void load_chunk(const Rows& R, int K, int sc, int p, uint64_t pol,
                                           uint32_t (&w)[16]) {
  const uint8_t* a = R.w + sc * kSC + p * 128;
  ld_w8(a, pol, w);
  ld_w8(a + (size_t)R.dr * K, pol, w + 8);
}

// 8 mma of one 128-column chunk: two chains, A from the code words of rows
// g (w[0..7]) and g + 8 (w[8..15]), B from x words xa (mma 0..3), xb (4..7)
__device__ __forceinline__ void chunk_mma(const uint32_t (&w)[16], const uint4& x0, const uint4& x1,
                                          const uint4& x2, const uint4& x3, float (&d0)[4],
                                          float (&d1)[4]) {
  mma_f16(d0, codes01(w[0]), codes01(w[8]), codes23(w[0]), codes23(w[8]), x0.x, x0.y);
  mma_f16(d1, codes01(w[1]), codes01(w[9]), codes23(w[1]), codes23(w[9]), x0.z, x0.w);
  mma_f16(d0, codes01(w[2]), codes01(w[10]), codes23(w[2]), codes23(w[10]), x1.x, x1.y);
  mma_f16(d1, codes01(w[3]), codes01(w[11]), codes23(w[3]), codes23(w[11]), x1.z, x1.w);
  mma_f16(d0, codes01(w[4]), codes01(w[12]), codes23(w[4]), codes23(w[12]), x2.x, x2.y);
  mma_f16(d1, codes01(w[5]), codes01(w[13]), codes23(w[5]), codes23(w[13]), x2.z, x2.w);
  mma_f16(d0, codes01(w[6]), codes01(w[14]), codes23(w[6]), codes23(w[14]), x3.x, x3.y);
  mma_f16(d1, codes01(w[7]), codes01(w[15]), codes23(w[7]), codes23(w[15]), x3.z, x3.w);
}

// The GEMV of one launch, for a CTA of W warps (of a grid of gridDim.x CTAs,
// this one blockIdx.x) and the batch tile blockIdx.y (4 NT rows each). `wait()` runs once the first weight loads are in
// flight and before anything written upstream is read (the
// programmatic-dependent-launch trigger and wait). smem: gtc_smem(K, NT, W)
// bytes.
// BULK: the instantiation with the bulk copy of a bf16 x (below); without
// it the kernel carries none of that code (the batch-1 decode chain is
// sensitive to the kernel's size: instruction fetch stalls lead its profile)
template <int NT, int W, bool BULK, class Wait>
__device__ __forceinline__ void gemv_tc_body(const Params& P, uint8_t* smem, Wait&& wait) {
  constexpr int kWarps = W, kThreads = W * 32;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int K = P.K, Kg = K / 64, nsc = K / kSC;
  // S <= nsc gives every warp of a team at least one super-chunk, so all S
  // warps of the team meet at its named barrier once per block (a warp with
  // none would skip the loop and leave the others waiting)
  int S = P.S;
  while (S > 1 && S > nsc) S >>= 1;
  // batch tile of this CTA: rows [b0, b0 + Bt) of the launch's P.B
  const int b0 = blockIdx.y * 4 * NT, Bt = min(4 * NT, P.B - b0);
  const int xs = K + 8;  // fp16 row stride of x (pad: batch rows on other banks)
  // regions in floats, each a multiple of 4 (16 bytes): xh is read with
  // 16-byte loads, so it must start on a 16-byte boundary for any W
  constexpr int kRed = ((4 * NT + 1) * kWarps + 3) & ~3;
  float* red = reinterpret_cast<float*>(smem);                      // [4 NT + 1][kWarps]
  float* part = red + kRed;                                          // [2][kWarps][32][2 NT]
  float* gsum = part + 2 * kWarps * 32 * 2 * NT;                    // [4 NT][Kg]
  uint16_t* xh = reinterpret_cast<uint16_t*>(gsum + 4 * NT * Kg);   // [4 NT][xs]
  // one batch tile of 8 warps: each warp's second unit of work (a 16-row
  // block's super-chunk) is staged here before the wait, 16-byte piece q of
  // chunk p of lane l at ((p * 4 + q) * 32 + l) * 16 (conflict-free)
  constexpr bool kStage2 = NT == 1 && W == 8;
  uint8_t* stage2 = reinterpret_cast<uint8_t*>(xh + 4 * NT * xs) + (size_t)warp * 8192;

  // L2 prefetch for a later kernel of the chain (one thread per CTA)
  if (tid == 0 && blockIdx.y == 0 && (P.pf.n > 0 || P.pf.kv.kc))
    issue_prefetch(P.pf, blockIdx.x, gridDim.x);

  // team = S warps sharing each block's columns; team slots are numbered
  // across CTAs first so that few blocks spread over many SMs
  const int tpc = kWarps / S, tl = warp / S, pw = warp % S;
  const int T = gridDim.x * tpc, team = tl * gridDim.x + blockIdx.x;
  const int sc_lo = pw * nsc / S, sc_hi = (pw + 1) * nsc / S, nscw = sc_hi - sc_lo;
  const int nblk = team < P.nblocks ? (P.nblocks - 1 - team) / T + 1 : 0;
  const int total = nscw > 0 ? nblk * nscw : 0;

  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));

  // the first loads go out before waiting for the previous kernel: weights
  // never depend on it
  uint32_t wb[4][16];
  uint32_t sv[4] = {0u, 0u, 0u, 0u};
  int lblk = team, lsc = sc_lo;  // position of the next super-chunk to load
  Rows lr = {};
  if (total > 0) {
    lr = rows_of(P, lblk, g, t);
    load_scales(lr, Kg, lsc, sv);
#pragma unroll
    for (int p = 0; p < 4; ++p) load_chunk(lr, K, lsc, p, pol, wb[p]);
  }
  // the second unit's codes go to shared memory and its scales to registers,
  // also before the wait, so that no weight load is left after it for a warp
  // with two units (K = 3072 split over teams of 4: the down projection)
  bool staged = false;
  uint32_t sv1[4] = {0u, 0u, 0u, 0u};
  if constexpr (kStage2) {
    if (total >= 2) {
      int sc1 = lsc + 1, blk1 = lblk;
      if (sc1 == sc_hi) {
        sc1 = sc_lo;
        blk1 += T;
      }
      const Rows r1 = rows_of(P, blk1, g, t);
      load_scales(r1, Kg, sc1, sv1);
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const uint8_t* a = r1.w + sc1 * kSC + p * 128;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint8_t* src = a + (q >> 1) * (size_t)r1.dr * K + (q & 1) * 16;
          const uint32_t dst = (uint32_t)__cvta_generic_to_shared(stage2 + ((p * 4 + q) * 32 + lane) * 16);
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
        }
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
      staged = true;
    }
  }

  // The input is formed in items of 128 columns of one batch row (lane l
  // holds columns 4l .. 4l + 3; lanes 0-15 cover one 64-column group, lanes
  // 16-31 the next); warp w forms items w, w + W, ... The first kItems of a
  // warp stay in registers from one load round to the forming pass (later
  // ones, for large B * K, are loaded again).
  constexpr int kItems = 3;
  const int Kp = K / 128, nitems = Bt * Kp;
  const int my_items = warp < nitems ? (nitems - 1 - warp) / kWarps + 1 : 0;
  auto nw_of = [&](int c) {  // (the norm weight may be only 2-byte aligned)
    return make_uint2((uint32_t)P.nw[c] | ((uint32_t)P.nw[c + 1] << 16),
                      (uint32_t)P.nw[c + 2] | ((uint32_t)P.nw[c + 3] << 16));
  };
  uint2 nwr[kItems];  // RMSNorm weights of the kept items (bf16 x 4)
#pragma unroll
  for (int j = 0; j < kItems; ++j) {
    nwr[j] = make_uint2(0u, 0u);
    if ((P.xmode == kXRmsNorm || P.xmode == kXRmsNormParts) && j < my_items)
      nwr[j] = nw_of(((warp + j * kWarps) % Kp) * 128 + 4 * lane);
  }

  wait();  // x (and residuals) are written upstream
  // what the previous kernels wrote (x, the residual) is read through L2
  // (ld.global.cg): each value is read once per CTA, so L1 would not help.
  // One round of loads: the kept input items and this warp's first residual
  // values, all in flight together. In SiLU mode an item holds silu(gate) *
  // up, not yet rounded.
  auto load_item = [&](int i) -> float4 {
    const int b = i / Kp, c = (i - b * Kp) * 128 + 4 * lane;
    const size_t o = (size_t)(b0 + b) * K + c;
    if (P.xmode == kXBf16) {
      const uint2 w2 = __ldcg(reinterpret_cast<const uint2*>(P.x + o));
      return make_float4(bf16_lo(w2.x), bf16_hi(w2.x), bf16_lo(w2.y), bf16_hi(w2.y));
    }
    float4 va = __ldcg(reinterpret_cast<const float4*>(P.xa + o));
    if (P.xmode == kXRmsNormParts) {
      const float* pb = P.parts + ((size_t)(b0 + b) * P.nparts) * K + c;
      for (int j = 0; j < P.nparts; ++j) {
        const float4 pj = __ldcg(reinterpret_cast<const float4*>(pb + (size_t)j * K));
        va.x += pj.x;
        va.y += pj.y;
        va.z += pj.z;
        va.w += pj.w;
      }
      if (blockIdx.x == 0) *reinterpret_cast<float4*>(P.xsum + o) = va;
    }
    if (P.xmode == kXSiluMul) {
      const float4 u = __ldcg(reinterpret_cast<const float4*>(P.xb + o));
      va = make_float4(va.x / (1.0f + expf(-va.x)) * u.x, va.y / (1.0f + expf(-va.y)) * u.y,
                       va.z / (1.0f + expf(-va.z)) * u.z, va.w / (1.0f + expf(-va.w)) * u.w);
    }
    return va;
  };
  // A bf16 x with more items than the warps keep in registers (large B x
  // K) goes to shared memory in bulk instead: 16-byte copies, four in flight
  // a thread, then an in-place conversion to fp16 (the item path would load
  // and form those items one dependent round at a time)
  const bool bulk = BULK && P.xmode == kXBf16 && nitems > kItems * kWarps &&
                    (reinterpret_cast<uintptr_t>(P.x) & 15) == 0;
  float4 xv[kItems];
#pragma unroll
  for (int j = 0; j < kItems; ++j)
    xv[j] = !bulk && j < my_items ? load_item(warp + j * kWarps) : make_float4(0.f, 0.f, 0.f, 0.f);
  // residual of the first block this warp stores (lane (g, t): rows g, g + 8
  // of batch row 4 nt + t)
  float resv[NT][2];
  const bool stores = total > 0 && (S == 1 || pw == 0);
  {
    const Seg& Sg = P.seg[seg_of(P, min(team, P.nblocks - 1))];
    const int row0 = (team - Sg.blk0) * kRB;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int b = 4 * nt + t, r = row0 + g + 8 * h;
        resv[nt][h] = 0.f;
        if (stores && Sg.res && b < Bt && r < Sg.N)
          resv[nt][h] = __ldcg(Sg.res + (size_t)(b0 + b) * Sg.N + r);
      }
    }
  }

  // 1) RMSNorm statistics per batch row: per lane over its items, then the
  // warp, then the warps in order (deterministic)
  float inv[4 * NT];
#pragma unroll
  for (int b = 0; b < 4 * NT; ++b) inv[b] = 0.f;
  const bool norm = P.xmode == kXRmsNorm || P.xmode == kXRmsNormParts;
  if (norm) {
    float ssb[4 * NT];
#pragma unroll
    for (int b = 0; b < 4 * NT; ++b) ssb[b] = 0.f;
    auto stat = [&](int i, const float4& v) {
      const int b = i / Kp;
      const float ss = fmaf(v.w, v.w, fmaf(v.z, v.z, fmaf(v.y, v.y, v.x * v.x)));
#pragma unroll
      for (int bb = 0; bb < 4 * NT; ++bb)
        if (b == bb) ssb[bb] += ss;
    };
#pragma unroll
    for (int j = 0; j < kItems; ++j)
      if (j < my_items) stat(warp + j * kWarps, xv[j]);
    for (int j = kItems; j < my_items; ++j) stat(warp + j * kWarps, load_item(warp + j * kWarps));
#pragma unroll
    for (int b = 0; b < 4 * NT; ++b) {
      const float ss = warp_sum(ssb[b]);
      if (lane == 0) red[b * kWarps + warp] = ss;
    }
    __syncthreads();
#pragma unroll
    for (int b = 0; b < 4 * NT; ++b) {
      if (b >= Bt) break;
      float ss = 0.f;
      for (int w = 0; w < kWarps; ++w) ss += red[b * kWarps + w];
      inv[b] = 1.0f / sqrtf(ss / (float)K + P.eps);
    }
  }
  // 2) the input values rounded to bf16 where the separate kernels round
  // them go to xh as fp16 and each 64-column group's fp16 sum to gsum. fp16
  // holds them exactly unless max|x| >= 2^15, checked after the pass; then
  // (rarely) the pass is redone on x * 2^-e. Batch rows past B are never
  // read by a live B lane.
  auto form_item = [&](int i, const float4& va, const uint2& nw2, float down) -> float {
    const int b = i / Kp, c = (i - b * Kp) * 128 + 4 * lane;
    float v[4] = {va.x, va.y, va.z, va.w};
    if (norm) {
      float ib = inv[0];
#pragma unroll
      for (int jb = 1; jb < 4 * NT; ++jb)
        if (b == jb) ib = inv[jb];
      const float wv[4] = {bf16_lo(nw2.x), bf16_hi(nw2.x), bf16_lo(nw2.y), bf16_hi(nw2.y)};
#pragma unroll
      for (int e = 0; e < 4; ++e) v[e] = v[e] * ib * wv[e];
    }
    float m = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[e] = bf16_bits_to_f32(f32_to_bf16_bits(v[e]));  // no-op for bf16 input
      m = fmaxf(m, fabsf(v[e]));
    }
    const size_t o = (size_t)(b0 + b) * K + c;
    if (P.xout && blockIdx.x == 0 && down == 1.0f)
      *reinterpret_cast<uint2*>(P.xout + o) =
          make_uint2((uint32_t)f32_to_bf16_bits(v[0]) | ((uint32_t)f32_to_bf16_bits(v[1]) << 16),
                     (uint32_t)f32_to_bf16_bits(v[2]) | ((uint32_t)f32_to_bf16_bits(v[3]) << 16));
    const __half2 h01 = __floats2half2_rn(v[0] * down, v[1] * down);
    const __half2 h23 = __floats2half2_rn(v[2] * down, v[3] * down);
    *reinterpret_cast<uint2*>(xh + b * xs + c) =
        make_uint2(*reinterpret_cast<const uint32_t*>(&h01), *reinterpret_cast<const uint32_t*>(&h23));
    // the 64-column group's sum over its 16 lanes (fixed order)
    float sum = (__low2float(h01) + __high2float(h01)) + (__low2float(h23) + __high2float(h23));
#pragma unroll
    for (int off = 8; off >= 1; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if ((lane & 15) == 0) gsum[b * Kg + c / 64] = sum;
    return m;
  };
  auto form = [&](float down) -> float {
    float mloc = 0.f;
#pragma unroll
    for (int j = 0; j < kItems; ++j)
      if (j < my_items) mloc = fmaxf(mloc, form_item(warp + j * kWarps, xv[j], nwr[j], down));
    for (int j = kItems; j < my_items; ++j) {
      const int i = warp + j * kWarps;
      const uint2 nw2 = norm ? nw_of((i % Kp) * 128 + 4 * lane) : make_uint2(0u, 0u);
      mloc = fmaxf(mloc, form_item(i, load_item(i), nw2, down));
    }
    return mloc;
  };
  // bulk: x's bf16 rows copied as they are into xh; returns this thread's max|x|
  auto bulk_copy = [&]() -> float {
    const int vpr = K / 8, nvec = Bt * vpr;
    float m = 0.f;
    for (int i0 = tid; i0 < nvec; i0 += kThreads * 4) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * kThreads;
        v[u] = make_uint4(0u, 0u, 0u, 0u);
        if (i < nvec)
          v[u] = __ldcg(reinterpret_cast<const uint4*>(P.x + (size_t)(b0 + i / vpr) * K) + i % vpr);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * kThreads;
        if (i < nvec) {
          *reinterpret_cast<uint4*>(xh + (i / vpr) * xs + (i % vpr) * 8) = v[u];
          const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
          for (int k = 0; k < 4; ++k) m = fmaxf(m, fmaxf(fabsf(bf16_lo(w[k])), fabsf(bf16_hi(w[k]))));
        }
      }
    }
    return m;
  };
  // bulk: xh converted in place to fp16 x * down, and each 64-column
  // group's fp16 sum to gsum; eight lanes a group (lane & 7: its 16-byte
  // chunk), the sum over them in a fixed order
  auto bulk_convert = [&](float down) {
    const int ng = Bt * Kg;
    for (int gi0 = warp * 4; gi0 < ng; gi0 += kWarps * 4) {
      const int gi = gi0 + (lane >> 3), c8 = lane & 7;
      float sum = 0.f;
      if (gi < ng) {
        uint4* p = reinterpret_cast<uint4*>(xh + (gi / Kg) * xs + (gi % Kg) * 64 + c8 * 8);
        const uint4 w = *p;
        uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const __half2 h = __floats2half2_rn(bf16_lo(ww[k]) * down, bf16_hi(ww[k]) * down);
          ww[k] = *reinterpret_cast<const uint32_t*>(&h);
          sum += __low2float(h) + __high2float(h);
        }
        *p = make_uint4(ww[0], ww[1], ww[2], ww[3]);
      }
      sum += __shfl_xor_sync(0xffffffffu, sum, 1);
      sum += __shfl_xor_sync(0xffffffffu, sum, 2);
      sum += __shfl_xor_sync(0xffffffffu, sum, 4);
      if (c8 == 0 && gi < ng) gsum[gi] = sum;  // gsum [4 NT][Kg]: row b at b Kg
    }
  };
  float mx = bulk ? bulk_copy() : form(1.0f);
  for (int i = Bt * Kg + tid; i < 4 * NT * Kg; i += kThreads) gsum[i] = 0.f;
  // 3) max|x| over the CTA; prescale 2^-e so that max|x| * 2^-e < 2^15
  mx = warp_max(mx);
  float* redm = red + 4 * NT * kWarps;
  if (lane == 0) redm[warp] = mx;
  __syncthreads();
  mx = 0.f;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) mx = fmaxf(mx, redm[w]);
  int e = 0;  // NaN or inf in x propagate to y without a prescale
  if (mx >= 32768.f && mx <= 3.0e38f) e = (int)ceilf(log2f(mx / 16384.f));
  const float up = exp2f((float)e);
  if (bulk) {  // (uniform over the CTA) xh holds the raw copy until here
    bulk_convert(exp2f((float)-e));
    __syncthreads();
  } else if (e != 0) {  // uniform over the CTA
    form(exp2f((float)-e));
    __syncthreads();
  }

  // B-operand lanes: column n = g = 2 b + h, live on the k-slots of group h
  bool xl[NT];
  const uint16_t* xrow[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int b = 4 * nt + (g >> 1);
    xl[nt] = b < Bt && (t >> 1) == (g & 1);
    xrow[nt] = xh + b * xs + 32 * t;
  }

  float acc[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = 0.f;
  int cblk = team, csc = sc_lo, nb = 0;
  for (int it = 0; it < total; ++it) {
    const bool more = it + 1 < total;
    if (more) {
      if (++lsc == sc_hi) {
        lsc = sc_lo;
        lblk += T;
        lr = rows_of(P, lblk, g, t);
      }
    }
    uint32_t svn[4] = {0u, 0u, 0u, 0u};
    const bool from_stage = staged && it == 0;  // the next unit is already in shared memory
    if (from_stage) {
#pragma unroll
      for (int i = 0; i < 4; ++i) svn[i] = sv1[i];
    } else if (more) {
      load_scales(lr, Kg, lsc, svn);
    }
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const int src = (lane & ~3) | p;
      const uint32_t s0 = __shfl_sync(0xffffffffu, sv[0], src);
      const uint32_t s1 = __shfl_sync(0xffffffffu, sv[1], src);
      const uint32_t b0 = __shfl_sync(0xffffffffu, sv[2], src);
      const uint32_t b1 = __shfl_sync(0xffffffffu, sv[3], src);
      // (scale, bias + 128 scale) of rows g, g+8 for groups A, B of the chunk
      const float sA0 = bf16_lo(s0), sB0 = bf16_hi(s0), sA1 = bf16_lo(s1), sB1 = bf16_hi(s1);
      const float cA0 = fmaf(128.f, sA0, bf16_lo(b0)), cB0 = fmaf(128.f, sB0, bf16_hi(b0));
      const float cA1 = fmaf(128.f, sA1, bf16_lo(b1)), cB1 = fmaf(128.f, sB1, bf16_hi(b1));
      const int chunk = csc * 4 + p;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        uint4 x0 = make_uint4(0u, 0u, 0u, 0u), x1 = x0, x2 = x0, x3 = x0;
        if (xl[nt]) {
          const uint4* xp = reinterpret_cast<const uint4*>(xrow[nt] + chunk * 128);
          x0 = xp[0];
          x1 = xp[1];
          x2 = xp[2];
          x3 = xp[3];
        }
        float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
        chunk_mma(wb[p], x0, x1, x2, x3, d0, d1);
        // lane (g, t): batch 4 nt + t; [0] row g group A, [1] row g group B,
        // [2] row g+8 group A, [3] row g+8 group B
        const float2 gs = *reinterpret_cast<const float2*>(gsum + (4 * nt + t) * Kg + 2 * chunk);
        acc[nt][0] = fmaf(sA0, d0[0] + d1[0], fmaf(cA0, gs.x, fmaf(sB0, d0[1] + d1[1],
                                                                   fmaf(cB0, gs.y, acc[nt][0]))));
        acc[nt][1] = fmaf(sA1, d0[2] + d1[2], fmaf(cA1, gs.x, fmaf(sB1, d0[3] + d1[3],
                                                                   fmaf(cB1, gs.y, acc[nt][1]))));
      }
      if (more && !from_stage) load_chunk(lr, K, lsc, p, pol, wb[p]);
    }
    if (from_stage) {
      asm volatile("cp.async.wait_all;" ::: "memory");
#pragma unroll
      for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 v = *reinterpret_cast<const uint4*>(stage2 + ((p * 4 + q) * 32 + lane) * 16);
          wb[p][q * 4 + 0] = v.x;
          wb[p][q * 4 + 1] = v.y;
          wb[p][q * 4 + 2] = v.z;
          wb[p][q * 4 + 3] = v.w;
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) sv[i] = svn[i];

    if (++csc < sc_hi) continue;
    // ------------------------------------------------ block done: store
    bool store = true;
    if (S > 1) {
      // partial sums of the team meet in shared memory (double-buffered by
      // block parity, one named barrier per block), summed in part order
      float* pb = part + (((nb & 1) * kWarps + tl * S) * 32) * 2 * NT;
      if (pw != 0) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          pb[((pw * 32) + lane) * 2 * NT + 2 * nt] = acc[nt][0];
          pb[((pw * 32) + lane) * 2 * NT + 2 * nt + 1] = acc[nt][1];
        }
      }
      asm volatile("bar.sync %0, %1;" ::"r"(1 + tl), "r"(S * 32) : "memory");
      if (pw == 0) {
        for (int q = 1; q < S; ++q) {
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            acc[nt][0] += pb[((q * 32) + lane) * 2 * NT + 2 * nt];
            acc[nt][1] += pb[((q * 32) + lane) * 2 * NT + 2 * nt + 1];
          }
        }
      } else {
        store = false;
      }
    }
    if (store) {
      const Seg& Sg = P.seg[seg_of(P, cblk)];
      const int row0 = (cblk - Sg.blk0) * kRB;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int b = 4 * nt + t;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int r = row0 + g + 8 * h;
          if (b < Bt && r < Sg.N) {
            const size_t o = (size_t)(b0 + b) * Sg.N + r;
            float v = acc[nt][h] * up;
            if (Sg.res) v += nb == 0 ? resv[nt][h] : __ldcg(Sg.res + o);
            if (Sg.y_bf16)
              reinterpret_cast<uint16_t*>(Sg.y)[o] = f32_to_bf16_bits(v);
            else
              reinterpret_cast<float*>(Sg.y)[o] = v;
          }
        }
      }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = 0.f;
    csc = sc_lo;
    cblk += T;
    ++nb;
  }
}

}  // namespace gtc

// dynamic shared memory of gemv_tc_body
inline size_t gtc_smem(int K, int NT, int W) {
  return (size_t)(((4 * NT + 1) * W + 3) & ~3) * 4 + (size_t)2 * W * 32 * 2 * NT * 4 +
         (size_t)4 * NT * (K / 64) * 4 + (size_t)4 * NT * (K + 8) * 2 +
         (NT == 1 && W == 8 ? (size_t)W * 8192 : 0);  // the second unit's staging
}

// Columns of each 16-row block are split over S warps (1, 2, 4, ... <= W,
// at most one 512-column super-chunk of work per warp beyond the first
// split) while the launch still has idle warp slots: a matrix of a decode
// layer then has all its weights in flight before the kernel waits for its
// input.
__host__ __device__ inline int gtc_split(int nblocks, int K, int W, int sms) {
  const int nsc = K / gtc::kSC;
  int S = 1;
  while (2 * S <= W && 2 * S <= nsc && (long long)nblocks * 2 * S <= (long long)sms * W) S *= 2;
  return S;
}

}  // namespace qg
