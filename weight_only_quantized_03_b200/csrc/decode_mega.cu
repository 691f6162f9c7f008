// Persistent decode-step kernel: one cooperative launch runs every layer of
// the Qwen3 decode step (turbospark-runtime 0.3.0, src/qwen3_asr_metal.rs,
// `step`: input norm -> q,k,v -> per-head q/k norm -> RoPE -> K/V append ->
// attention over [0, position] -> o_proj + residual -> post-attention norm
// -> gate, up -> SiLU-mul -> down + residual; final norm; tied LM head).
//
// Work layout
//   * One CTA per SM (cooperative launch: all CTAs co-resident): one
//     producer warp and kCW consumer warps.
//   * Every GEMV row block (16 rows) and attention chunk (32 KV rows) a CTA
//     touches is fixed by (CTA index, config, sequence lengths). The
//     producer walks that schedule once for the whole step and streams each
//     tile -- 16 rows x up to 1024 packed columns with their scales and
//     biases, one bulk copy per row into a padded (bank-conflict-free)
//     layout, or a K and V chunk -- from HBM into a ring of shared-memory
//     stages with cp.async.bulk, completing on an mbarrier. It waits only for
//     a free stage, never for activations, so weight streaming runs ahead
//     through the phase boundaries.
//   * Consumers walk the same schedule (the same `walk`) and consume tiles.
//
// GEMV on the tensor cores (mma.sync m16n8k16, bf16 in, fp32 accumulate):
//   A = 16 weight rows, each packed code byte q in [0, 255] converted exactly
//   to bf16; B = up to 8 activation columns (the sequences), bf16 as stored.
//   The k order inside an mma is permuted so that each thread's A bytes and B
//   values are contiguous in shared memory (the sum over k does not depend
//   on the order). Per group of 64 columns the mma result S_g = sum q x
//   becomes s_g * S_g + beta_g * sum_g(x) (the affine factorisation), in
//   fp32. The consumer warps split K; their partial sums are reduced through
//   shared memory once per row block.
//
// Exchanges between CTAs carry their own ready flag: each 64-bit word holds
// a 32-bit payload (fp32, or two bf16) and a 32-bit epoch (step counter,
// layer, phase), written and read with relaxed 64-bit accesses, so a
// consumer needs one L2 round trip and no separate counter. Each layer has
// its own exchange buffers, so nothing is rewritten within a step. Every
// wait is bounded (1 s); on expiry the kernel records an error word, skips
// the remaining work while still passing every barrier, and the producer
// waits (bounded) for its copies in flight before leaving.
#include <algorithm>
#include <cstring>

#include "qg_internal.cuh"

namespace qg {
namespace mk {

constexpr int kCW = 8;              // consumer warps
constexpr int kCT = kCW * 32;       // consumer threads
constexpr int kThreads = kCT + 32;  // + one producer warp
constexpr int kRB = 16;             // rows per GEMV block (mma M)
constexpr int kKc = 1024;           // columns per GEMV tile
constexpr int kCH = 32;             // KV rows per ring stage of an attention item
constexpr int kCHI = 128;           // KV rows per attention item (4 stages)
constexpr int kMaxLayers = 64;
constexpr int kMaxB = 4;
constexpr int kMaxG = 8;
constexpr int kMaxD = 128;
constexpr int kStageW = kRB * kKc;  // weight bytes of a stage (16 rows x 1024 columns)
// a stage also holds the row block's scales and biases (16 x K/64 each);
// its size is set at launch from the largest K
constexpr unsigned long long kWaitNs = 1000000000ull;
constexpr int kLog = 1024;

enum Kind { T_QKV = 0, T_ATTN, T_O, T_GATE, T_UP, T_DOWN, T_HEAD };
enum Phase { E_QKV = 1, E_ATT = 2, E_O = 4, E_UP = 5, E_DOWN = 6, E_NEVER = 7 };
enum { C_ERR = 0, C_START = 1 };  // counters, zeroed at the start of each step

struct Layer {
  const uint8_t* w[7];  // q k v o gate up down
  const uint16_t* s[7];
  const uint16_t* b[7];
  const uint16_t* in_norm;
  const uint16_t* post_norm;
  const uint16_t* q_norm;
  const uint16_t* k_norm;
};

struct Params {
  int hidden, nlayers, H, Hkv, D, ffn, vocab, B, cap, stages, stage_bytes, maxsplit;
  int test_stall;  // test hook: one wait targets a word that nothing writes
  float eps, scale;
  double theta;
  const uint8_t* ew;
  const uint16_t* es;
  const uint16_t* eb;
  const uint16_t* final_norm;
  uint16_t* kc;
  uint16_t* vc;
  const int32_t* tokens;
  const int32_t* positions;
  float* logits;
  float* x;                   // [B][hidden] final residual stream (fp32)
  unsigned* cnt;              // counters (zeroed each step)
  unsigned* step;             // step counter (persists across steps)
  unsigned long long* trace;  // optional [CTA][layer + 1][16] %globaltimer stamps
  unsigned long long* log;    // optional [CTA][kLog] (event << 56 | time) records
  // exchange words, one buffer per layer
  unsigned long long* xo;    // [L][B][hidden]              x after o_proj + residual
  unsigned long long* xd;    // [L][B][hidden]              x after down + residual
  unsigned long long* qkv;   // [L][B][qd + 2 kd]           q, k, v GEMV outputs
  unsigned long long* part;  // [L][B][H][maxsplit][D + 2]  item partials (o[D], max, sum)
  unsigned long long* hh;    // [L][B][ffn / 2]             SiLU-mul output, bf16 pairs
  Layer layer[kMaxLayers];
};

struct Tile {
  int kind, layer, seg, row0, nrows, K, kc, last, b, g, s, sub;
};

// ------------------------------------------------------------ helpers ----

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                         uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}
__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ unsigned long long ld_word(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_word(unsigned long long* p, unsigned payload, unsigned epoch) {
  const unsigned long long v = ((unsigned long long)epoch << 32) | payload;
  asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long now_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kCT) : "memory"); }
__device__ __forceinline__ void set_err(unsigned* cnt, unsigned code) { atomicCAS(cnt + C_ERR, 0u, code); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// code bytes (2i, 2i+1) of a word as a bf16 pair (exact: codes are integers <= 255)
template <int I>
__device__ __forceinline__ uint32_t codes_bf16x2(uint32_t w) {
  return pack_bf16x2(byte_to_f32<2 * I>(w), byte_to_f32<2 * I + 1>(w));
}

__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Bounded wait on a ring-stage barrier; false on timeout or error.
__device__ bool stage_wait(uint64_t* bar, uint32_t parity, unsigned* cnt, unsigned code) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = now_ns();
  for (unsigned i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63) == 0) {
      if (ld_acquire(cnt + C_ERR)) return false;
      if (now_ns() - t0 > kWaitNs) break;
    }
  }
  set_err(cnt, code);
  return false;
}

__device__ __forceinline__ int part_lo(int n, int c, int G) { return (int)((long long)n * c / G); }

// ---------------------------------------------------------- schedule ----

struct SeqInfo {
  int L[kMaxB];   // attended rows (0 when the sequence's token or position is invalid)
  int ns[kMaxB];  // attention items (128-row splits) per KV head
  int nitems;     // attention items (b, g, s) per layer
};

__device__ __forceinline__ void seq_info(const Params& P, SeqInfo& si) {
  si.nitems = 0;
  for (int b = 0; b < kMaxB; ++b) {
    si.L[b] = 0;
    si.ns[b] = 0;
    if (b >= P.B) continue;
    const int t = __ldg(P.tokens + b), p = __ldg(P.positions + b);
    if (t >= 0 && t < P.vocab && p >= 0 && p < P.cap) {
      si.L[b] = p + 1;
      si.ns[b] = (p + kCHI) / kCHI;
      si.nitems += P.Hkv * si.ns[b];
    }
  }
}

// Row blocks [blk0, blk1) of 16 rows of one matrix, in tiles of <= 1024 columns.
template <class F>
__device__ __forceinline__ void gemv_tiles(F& f, int kind, int l, int seg, int blk0, int blk1,
                                           int nrow_total, int K) {
  const int nkc = (K + kKc - 1) / kKc;
  for (int bk = blk0; bk < blk1; ++bk) {
    const int r = bk * kRB;
    const int n = min(kRB, nrow_total - r);
    for (int kc = 0; kc < nkc; ++kc)
      f.tile(Tile{kind, l, seg, r, n, K, kc, kc == nkc - 1 ? 1 : 0, 0, 0, 0, 0});
  }
}

// The fixed order of tiles and phase boundaries of this CTA. Producer and
// consumers run the same walk, so their stage sequences always agree. The
// walk always runs to the end; after a failed wait the functors only skip
// work, so every named barrier is reached by every consumer thread.
template <class F>
__device__ void walk(const Params& P, const SeqInfo& si, F& f) {
  const int c = blockIdx.x, G = gridDim.x;
  const int qd = P.H * P.D, kd = P.Hkv * P.D;
  const int bq = qd / kRB, bk = kd / kRB, bh = P.hidden / kRB, bf = P.ffn / kRB;
  const int nb_qkv = bq + 2 * bk;
  const int q0 = part_lo(nb_qkv, c, G), q1 = part_lo(nb_qkv, c + 1, G);
  const int h0 = part_lo(bh, c, G), h1 = part_lo(bh, c + 1, G);
  const int f0 = part_lo(bf, c, G), f1 = part_lo(bf, c + 1, G);
  for (int l = 0; l < P.nlayers; ++l) {
    f.begin(T_QKV, l);
    for (int b = q0; b < q1; ++b) {  // blocks of the concatenated [q; k; v] rows
      const int seg = b < bq ? 0 : (b < bq + bk ? 1 : 2);
      const int local = b - (seg == 0 ? 0 : (seg == 1 ? bq : bq + bk));
      gemv_tiles(f, T_QKV, l, seg, local, local + 1, seg == 0 ? qd : kd, P.hidden);
    }
    f.end(T_QKV, l);
    f.begin(T_ATTN, l);
    for (int i = c; i < si.nitems; i += G) {
      int j = i, b = 0;
      while (j >= P.Hkv * si.ns[b]) { j -= P.Hkv * si.ns[b]; ++b; }
      const int g = j / si.ns[b], s = j % si.ns[b];
      const int r1 = min(si.L[b], (s + 1) * kCHI);
      const int nsub = (r1 - s * kCHI + kCH - 1) / kCH;
      for (int u = 0; u < nsub; ++u) {
        const int r0 = s * kCHI + u * kCH;
        f.tile(Tile{T_ATTN, l, 0, r0, min(kCH, r1 - r0), 0, 0, u == nsub - 1 ? 1 : 0, b, g, s, u});
      }
    }
    f.end(T_ATTN, l);
    f.begin(T_O, l);
    gemv_tiles(f, T_O, l, 3, h0, h1, P.hidden, qd);
    f.end(T_O, l);
    f.begin(T_GATE, l);
    for (int b = f0; b < f1; ++b) {
      gemv_tiles(f, T_GATE, l, 4, b, b + 1, P.ffn, P.hidden);
      gemv_tiles(f, T_UP, l, 5, b, b + 1, P.ffn, P.hidden);
    }
    f.end(T_GATE, l);
    f.begin(T_DOWN, l);
    gemv_tiles(f, T_DOWN, l, 6, h0, h1, P.hidden, P.ffn);
    f.end(T_DOWN, l);
  }
  f.begin(T_HEAD, P.nlayers);
  const int bv = (P.vocab + kRB - 1) / kRB;
  gemv_tiles(f, T_HEAD, P.nlayers, 7, part_lo(bv, c, G), part_lo(bv, c + 1, G), P.vocab, P.hidden);
  f.end(T_HEAD, P.nlayers);
}

// --------------------------------------------------------- producer -----

struct Producer {
  const Params& P;
  uint8_t* ring;
  uint64_t* full;
  uint64_t* empty;
  uint64_t pol;
  int lane;
  int k = 0;
  bool dead = false;

  __device__ void begin(int, int) {}
  __device__ void end(int, int) {}

  __device__ void tile(const Tile& t) {
    if (dead) return;
    const int st = k % P.stages;
    const uint32_t par = (uint32_t)(k / P.stages) & 1u;
    bool ok = true;
    if (lane == 0) ok = stage_wait(&empty[st], par ^ 1u, P.cnt, 0x100u | (unsigned)t.kind);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    if (!ok) {
      dead = true;  // issue nothing more; the consumers' waits give up too
      return;
    }
    uint8_t* dst = ring + (size_t)st * P.stage_bytes;
    if (t.kind == T_ATTN) {
      if (lane == 0) {
        const size_t row = (((size_t)t.b * P.Hkv + t.g) * P.cap + t.row0) * P.D;
        const size_t lay = (size_t)t.layer * P.B * P.Hkv * P.cap * P.D;
        const uint32_t bytes = (uint32_t)t.nrows * P.D * 2;
        mbar_expect_tx(&full[st], 2 * bytes);
        bulk_g2s(dst, P.kc + lay + row, bytes, &full[st], pol);
        bulk_g2s(dst + kCH * kMaxD * 2, P.vc + lay + row, bytes, &full[st], pol);
      }
    } else {
      const uint8_t* w;
      const uint16_t* s;
      const uint16_t* b;
      if (t.kind == T_HEAD) {
        w = P.ew; s = P.es; b = P.eb;
      } else {
        const Layer& L = P.layer[t.layer];
        w = L.w[t.seg]; s = L.s[t.seg]; b = L.b[t.seg];
      }
      const int Kc = min(kKc, t.K - t.kc * kKc);
      // the block's scales and biases (all of its groups) ride with its first tile
      const uint32_t sb = t.kc == 0 ? (uint32_t)t.nrows * (t.K / 64) * 2 : 0u;
      if (lane == 0) mbar_expect_tx(&full[st], (uint32_t)t.nrows * Kc + 2 * sb);
      __syncwarp();
      if (Kc == t.K) {  // whole rows: the block is one contiguous run
        if (lane == 0) bulk_g2s(dst, w + (size_t)t.row0 * t.K, (uint32_t)t.nrows * t.K, &full[st], pol);
      } else if (lane < t.nrows) {  // one row segment per lane
        const size_t r = (size_t)t.row0 + lane;
        bulk_g2s(dst + lane * Kc, w + r * t.K + (size_t)t.kc * kKc, Kc, &full[st], pol);
      }
      if (sb && lane == 1) {
        uint8_t* sd = dst + kStageW;
        const size_t go = (size_t)t.row0 * (t.K / 64);
        bulk_g2s(sd, s + go, sb, &full[st], pol);
        bulk_g2s(sd + kRB * (t.K / 64) * 2, b + go, sb, &full[st], pol);
      }
    }
    __syncwarp();
    ++k;
  }

  // Before leaving: wait (bounded) until the copies of the last stages issued
  // have landed, so no bulk copy targets shared memory of an exited CTA.
  __device__ void drain() {
    if (lane != 0) return;
    const int lo = k - P.stages > 0 ? k - P.stages : 0;
    const unsigned long long t0 = now_ns();
    for (int j = lo; j < k; ++j) {
      const int st = j % P.stages;
      const uint32_t par = (uint32_t)(j / P.stages) & 1u;
      while (!mbar_try_wait(&full[st], par) && now_ns() - t0 < kWaitNs) {
      }
    }
  }
};

// --------------------------------------------------------- consumers ----

struct Smem {
  float* xstage;   // [kMaxB][hidden] fp32 residual stream (norm input)
  uint16_t* xin;   // [kMaxB][xs] bf16 GEMV input
  float* gsum;     // [kMaxB][gs] group sums of xin
  uint16_t* bsc;   // [2][kRB][Kmax/64] scales, biases of the current row block
  float* xown;     // [kMaxB][kRB] owned residual rows
  float* red;      // [kCW][kRB][8] split-K partials
  float* hbuf;     // [kRB][kMaxB] gate results, then SiLU-mul results
  float* rope;     // [kMaxB][kMaxD/2][2]
  float* qs;       // [kMaxG][kMaxD] normed, rotated, scaled q heads
  float* kv;       // [2][kMaxD] k and v rows of the current item (fp32)
  float* sc;       // [kMaxG][kCH] weights of the current stage, then [kMaxG] rescale factors
  float* ml;       // [kMaxB][H][maxsplit][2] item (max, sum) while merging
  int* flag;       // [8]
  int xs;          // row stride of xin (elements)
  int gs;          // row stride of gsum (groups)
};

struct Consumer {
  const Params& P;
  const SeqInfo& si;
  Smem S;
  uint8_t* ring;
  uint64_t* full;
  uint64_t* empty;
  unsigned base;  // epoch base of this step
  int k = 0;
  int tid = 0, warp = 0, lane = 0;
  int kin = 0;        // K of the current GEMV input in xin
  bool dead = false;  // a wait gave up: skip work, keep the barrier sequence
  float acc[4] = {0.f, 0.f, 0.f, 0.f};  // split-K partial of the current row block
  // running softmax state of the current attention item: warp h keeps the
  // running max and sum of query head h (h < Gq <= kCW); element e of
  // thread tid is output (h, d) with h * D + d = tid + e * kCT.
  static constexpr int kPer = kMaxG * kMaxD / kCT;
  float hm = -INFINITY, hl = 0.f;
  float ao[kPer];

  __device__ unsigned epoch(int l, int ph) const { return base + (unsigned)(l * 8 + ph); }

  int nlog = 0;
  __device__ void stamp(int l, int ev) {
    if (P.trace && tid == 0)
      P.trace[((size_t)blockIdx.x * (P.nlayers + 1) + l) * 16 + ev] = now_ns();
  }
  __device__ void log(unsigned ev) {
    if (P.log && tid == 0 && nlog < kLog)
      P.log[(size_t)blockIdx.x * kLog + nlog++] = ((unsigned long long)ev << 56) | (now_ns() & 0xFFFFFFFFFFFFull);
  }

  // CTA-uniform "every consumer thread succeeded" (all consumer threads call it).
  __device__ bool all_ok(bool ok) {
    if (tid == 0) S.flag[0] = 1;
    consumer_sync();
    if (!ok) S.flag[0] = 0;
    consumer_sync();
    const bool r = S.flag[0] != 0;
    consumer_sync();
    if (!r) dead = true;
    return r;
  }

  // Spin (bounded) until word w carries epoch ep; `v` holds the last value read.
  // After a few quick re-reads the spin backs off, so that many waiting
  // threads do not crowd the L2 slices the producers are writing to.
  __device__ bool spin_word(const unsigned long long* w, unsigned ep, unsigned long long& v,
                            unsigned code) {
    if ((unsigned)(v >> 32) == ep) return true;
    if (dead) return false;
    const unsigned long long t0 = now_ns();
    for (unsigned i = 1;; ++i) {
      v = ld_word(w);
      if ((unsigned)(v >> 32) == ep) return true;
      if (i > 2) __nanosleep(i < 16 ? 64 : 256);
      if ((i & 15) == 0) {
        if (ld_acquire(P.cnt + C_ERR)) break;
        if (now_ns() - t0 > kWaitNs) {
          set_err(P.cnt, code);
          break;
        }
      }
    }
    dead = true;
    return false;
  }

  // Read words addr(i) for i = tid, tid + kCT, ... < n (a batch of loads
  // issued before any wait), wait for epoch ep, hand payloads to put(i, v).
  template <class A, class F>
  __device__ bool poll_at(int n, A&& addr, unsigned ep, unsigned code, F&& put) {
    constexpr int kBatch = 8;
    bool ok = !dead;
    for (int i0 = tid; i0 < n; i0 += kBatch * kCT) {
      unsigned long long v[kBatch];
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const int i = i0 + j * kCT;
        v[j] = (ok && i < n) ? ld_word(addr(i)) : 0ull;
      }
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const int i = i0 + j * kCT;
        if (i < n) {
          if (ok) ok = spin_word(addr(i), ep, v[j], code);
          put(i, (unsigned)v[j]);
        }
      }
    }
    return ok;
  }

  template <class F>
  __device__ bool poll(const unsigned long long* src, int n, unsigned ep, unsigned code, F&& put) {
    return poll_at(n, [&](int i) { return src + i; }, ep, code, put);
  }

  // Block-wide sum over the consumer threads.
  __device__ float block_sum(float v) {
    v = warp_sum(v);
    consumer_sync();
    if (lane == 0) S.red[warp] = v;
    consumer_sync();
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kCW; ++w) t += S.red[w];
    consumer_sync();
    return t;
  }

  // xin[b] = bf16(rmsnorm(xstage[b]) * w), then the group sums.
  __device__ void norm_to_xin(const uint16_t* w) {
    const int n = P.hidden;
    for (int b = 0; b < P.B; ++b) {
      const float* xr = S.xstage + b * n;
      float ss = 0.f;
      for (int i = tid; i < n; i += kCT) ss = fmaf(xr[i], xr[i], ss);
      ss = block_sum(ss);
      const float inv = 1.0f / sqrtf(ss / (float)n + P.eps);
      for (int i = tid; i < n; i += kCT)
        S.xin[b * S.xs + i] = f32_to_bf16_bits(xr[i] * inv * bf16_bits_to_f32(__ldg(w + i)));
    }
    kin = n;
    consumer_sync();
    group_sums();
  }

  __device__ void group_sums() {
    const int ng = kin >> 6;
    for (int i = tid; i < P.B * ng; i += kCT) {
      const int b = i / ng, gi = i % ng;
      const uint4* p = reinterpret_cast<const uint4*>(S.xin + b * S.xs + 64 * gi);
      float s = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint4 u = p[j];
        s += bf16_lo(u.x) + bf16_hi(u.x) + bf16_lo(u.y) + bf16_hi(u.y) + bf16_lo(u.z) +
             bf16_hi(u.z) + bf16_lo(u.w) + bf16_hi(u.w);
      }
      S.gsum[b * S.gs + gi] = s;
    }
    consumer_sync();
  }

  // fp32 words [B][hidden] -> xstage
  __device__ void poll_x(const unsigned long long* src, unsigned ep, unsigned code) {
    log(10);
    float* xs = S.xstage;
    const bool ok = poll(src, P.B * P.hidden, ep, code,
                         [&](int i, unsigned v) { xs[i] = __uint_as_float(v); });
    all_ok(ok);
    log(11);
  }

  // bf16-pair words [B][K/2] -> xin, then the group sums
  __device__ void poll_bf16(const unsigned long long* src, int K, unsigned ep, unsigned code) {
    const int hw = K / 2;
    uint16_t* xin = S.xin;
    const int xs = S.xs;
    const bool ok = poll(src, P.B * hw, ep, code, [&](int i, unsigned v) {
      reinterpret_cast<uint32_t*>(xin + (i / hw) * xs)[i % hw] = v;
    });
    kin = K;
    all_ok(ok);
    group_sums();
  }

  __device__ void embed_to_xstage() {
    const int n = P.hidden;
    for (int i = tid; i < P.B * n; i += kCT) {
      const int b = i / n, c = i % n;
      float val;
      if (si.L[b] == 0) {
        val = __int_as_float(0x7fc00000);
      } else {
        const int t = __ldg(P.tokens + b);
        const float q = (float)__ldg(P.ew + (size_t)t * n + c);
        const size_t g = (size_t)t * (n / 64) + c / 64;
        val = fmaf(q, bf16_bits_to_f32(__ldg(P.es + g)), bf16_bits_to_f32(__ldg(P.eb + g)));
      }
      S.xstage[i] = val;
    }
    consumer_sync();
  }

  // a CTA owns at most one 16-row block of the residual stream
  __device__ void own_from_xstage() {
    const int bh = P.hidden / kRB;
    const int b0 = part_lo(bh, blockIdx.x, gridDim.x), b1 = part_lo(bh, blockIdx.x + 1, gridDim.x);
    if (b1 > b0)
      for (int i = tid; i < P.B * kRB; i += kCT)
        S.xown[i] = S.xstage[(i / kRB) * P.hidden + b0 * kRB + i % kRB];
    consumer_sync();
  }

  // Attention output of layer l for every sequence and head: merge the
  // items' partials (split order; the result does not depend on timing) and
  // write it to xin as bf16 (the o_proj input), then the group sums.
  __device__ void merge_attention(int l, bool stall) {
    log(5);
    const int D = P.D, H = P.H, ms = P.maxsplit;
    const unsigned ep = epoch(l, stall ? E_NEVER : E_ATT);
    bool ok = true;
    for (int b = 0; b < P.B; ++b) {
      const int ns = si.ns[b];
      const unsigned long long* pb = P.part + (((size_t)l * P.B + b) * H) * ms * (D + 2);
      float* ml = S.ml;
      // (max, sum) of every item of sequence b
      ok = poll_at(
               H * ns * 2,
               [&](int i) { return pb + ((size_t)((i >> 1) / ns) * ms + (i >> 1) % ns) * (D + 2) + D + (i & 1); },
               ep, 0x300u, [&](int i, unsigned v) { ml[i] = __uint_as_float(v); }) &&
           ok;
      consumer_sync();
      log(6);
      // one output pair (h, d..d+1) per thread; the items' o words loaded together
      for (int i = tid; i < H * D / 2; i += kCT) {
        const int h = i / (D / 2), d = 2 * (i % (D / 2));
        float M = -INFINITY;
        for (int j = 0; j < ns; ++j) M = fmaxf(M, ml[(h * ns + j) * 2]);
        float Ls = 0.f, O0 = 0.f, O1 = 0.f;
        for (int j0 = 0; j0 < ns; j0 += 8) {
          unsigned long long v[16];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const unsigned long long* pj = pb + ((size_t)h * ms + j0 + j) * (D + 2) + d;
            v[2 * j] = (ok && j0 + j < ns) ? ld_word(pj) : 0ull;
            v[2 * j + 1] = (ok && j0 + j < ns) ? ld_word(pj + 1) : 0ull;
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (j0 + j < ns) {
              const unsigned long long* pj = pb + ((size_t)h * ms + j0 + j) * (D + 2) + d;
              if (ok)
                ok = spin_word(pj, ep, v[2 * j], 0x301u) && spin_word(pj + 1, ep, v[2 * j + 1], 0x302u);
              const float e = expf(ml[(h * ns + j0 + j) * 2] - M);
              Ls = fmaf(ml[(h * ns + j0 + j) * 2 + 1], e, Ls);
              O0 = fmaf(__uint_as_float((unsigned)v[2 * j]), e, O0);
              O1 = fmaf(__uint_as_float((unsigned)v[2 * j + 1]), e, O1);
            }
          }
        }
        const float r0 = ns ? O0 / Ls : 0.f, r1 = ns ? O1 / Ls : 0.f;
        reinterpret_cast<uint32_t*>(S.xin + b * S.xs)[(h * D + d) / 2] =
            (uint32_t)f32_to_bf16_bits(r0) | ((uint32_t)f32_to_bf16_bits(r1) << 16);
      }
      consumer_sync();
    }
    kin = H * D;
    all_ok(ok);
    group_sums();
    log(7);
  }

  __device__ void begin(int kind, int l) {
    stamp(l, 2 * kind);
    const size_t xl = (size_t)P.B * P.hidden;
    switch (kind) {
      case T_QKV:
        if (l == 0)
          embed_to_xstage();
        else
          poll_x(P.xd + (l - 1) * xl, epoch(l - 1, E_DOWN), 0x200u);
        own_from_xstage();
        norm_to_xin(P.layer[l].in_norm);
        break;
      case T_O:
        merge_attention(l, P.test_stall && l == 0);
        break;
      case T_GATE:
        poll_x(P.xo + l * xl, epoch(l, E_O), 0x400u);
        norm_to_xin(P.layer[l].post_norm);
        break;
      case T_DOWN:
        poll_bf16(P.hh + (size_t)l * P.B * P.ffn / 2, P.ffn, epoch(l, E_UP), 0x500u);
        break;
      case T_HEAD:
        poll_x(P.xd + (P.nlayers - 1) * xl, epoch(P.nlayers - 1, E_DOWN), 0x600u);
        if (blockIdx.x == 0)
          for (int i = tid; i < P.B * P.hidden; i += kCT) P.x[i] = S.xstage[i];
        norm_to_xin(P.final_norm);
        break;
      default:
        break;
    }
    stamp(l, 2 * kind + 1);
  }

  __device__ void end(int kind, int l) { stamp(l, 14 + (kind == T_HEAD ? 1 : 0)); }

  // Per-warp bounded wait for the next stage; a warp that gives up stays dead.
  __device__ bool acquire_stage(int& st) {
    st = k % P.stages;
    const uint32_t par = (uint32_t)(k / P.stages) & 1u;
    bool ok = !dead;
    if (ok && lane == 0) ok = stage_wait(&full[st], par, P.cnt, 0x700u);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    if (!ok) dead = true;
    return ok;
  }

  __device__ void release_stage(int st) {
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
    ++k;
  }

  __device__ void tile(const Tile& t) {
    int st;
    const bool ok = acquire_stage(st);
    if (t.kind == T_HEAD) log(8);
    uint8_t* stage = ring + (size_t)st * P.stage_bytes;
    if (t.kind == T_ATTN) {
      attention(t, stage, ok);  // contains CTA barriers: always entered
      release_stage(st);
      return;
    }
    if (t.kc == 0) {
      // the row block's scales and biases, kept for all of its tiles
      acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
      const int n = t.nrows * (t.K / 64);  // bf16 values per array
      const uint16_t* src = reinterpret_cast<const uint16_t*>(stage + kStageW);
      for (int i = tid; ok && i < n; i += kCT) {
        S.bsc[i] = src[i];
        S.bsc[kRB * (t.K / 64) + i] = src[kRB * (t.K / 64) + i];
      }
      consumer_sync();
    }
    if (ok) gemv_tile(t, stage);
    release_stage(st);
    if (t.last) finish_block(t);  // contains CTA barriers: always entered
    if (t.kind == T_HEAD) log(9);
  }

  // ---- one tile: 16 rows x Kc columns; this warp's 64-column groups into acc
  __device__ void gemv_tile(const Tile& t, const uint8_t* stage) {
    const int Kc = min(kKc, t.K - t.kc * kKc);
    const int ng = Kc / 64, Kg = t.K / 64;
    const int g = lane >> 2, q = lane & 3;
    const uint16_t* Sc = S.bsc;
    const uint16_t* Bi = S.bsc + kRB * Kg;
    for (int gi = warp; gi < ng; gi += kCW) {
      const uint4 ra = *reinterpret_cast<const uint4*>(stage + g * Kc + gi * 64 + 16 * q);
      const uint4 rb = *reinterpret_cast<const uint4*>(stage + (g + 8) * Kc + gi * 64 + 16 * q);
      uint4 x0 = make_uint4(0, 0, 0, 0), x1 = x0;
      const int col = t.kc * kKc + gi * 64 + 16 * q;
      if (g < P.B) {
        const uint4* xp = reinterpret_cast<const uint4*>(S.xin + g * S.xs + col);
        x0 = xp[0];
        x1 = xp[1];
      }
      float c[4] = {0.f, 0.f, 0.f, 0.f};
      mma_bf16(c, codes_bf16x2<0>(ra.x), codes_bf16x2<0>(rb.x), codes_bf16x2<1>(ra.x),
               codes_bf16x2<1>(rb.x), x0.x, x0.y);
      mma_bf16(c, codes_bf16x2<0>(ra.y), codes_bf16x2<0>(rb.y), codes_bf16x2<1>(ra.y),
               codes_bf16x2<1>(rb.y), x0.z, x0.w);
      mma_bf16(c, codes_bf16x2<0>(ra.z), codes_bf16x2<0>(rb.z), codes_bf16x2<1>(ra.z),
               codes_bf16x2<1>(rb.z), x1.x, x1.y);
      mma_bf16(c, codes_bf16x2<0>(ra.w), codes_bf16x2<0>(rb.w), codes_bf16x2<1>(ra.w),
               codes_bf16x2<1>(rb.w), x1.z, x1.w);
      const int gg = t.kc * (kKc / 64) + gi;
      const float s0 = bf16_bits_to_f32(Sc[g * Kg + gg]), s1 = bf16_bits_to_f32(Sc[(g + 8) * Kg + gg]);
      const float b0 = bf16_bits_to_f32(Bi[g * Kg + gg]), b1 = bf16_bits_to_f32(Bi[(g + 8) * Kg + gg]);
      const float xs0 = (2 * q < P.B) ? S.gsum[(2 * q) * S.gs + gg] : 0.f;
      const float xs1 = (2 * q + 1 < P.B) ? S.gsum[(2 * q + 1) * S.gs + gg] : 0.f;
      acc[0] = fmaf(s0, c[0], fmaf(b0, xs0, acc[0]));
      acc[1] = fmaf(s0, c[1], fmaf(b0, xs1, acc[1]));
      acc[2] = fmaf(s1, c[2], fmaf(b1, xs0, acc[2]));
      acc[3] = fmaf(s1, c[3], fmaf(b1, xs1, acc[3]));
    }
  }

  // ---- reduce the warps' partials of a row block and emit its outputs
  __device__ void finish_block(const Tile& t) {
    const int g = lane >> 2, q = lane & 3;
    float* rw = S.red + warp * kRB * 8;
    rw[g * 8 + 2 * q] = acc[0];
    rw[g * 8 + 2 * q + 1] = acc[1];
    rw[(g + 8) * 8 + 2 * q] = acc[2];
    rw[(g + 8) * 8 + 2 * q + 1] = acc[3];
    consumer_sync();
    if (tid < kRB * kMaxB) {
      const int r = tid / kMaxB, b = tid % kMaxB;
      if (r < t.nrows && b < P.B && !dead) {
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < kCW; ++w) v += S.red[w * kRB * 8 + r * 8 + b];
        emit(t, r, b, v);
      }
    }
    consumer_sync();
    if (t.kind == T_UP) {
      // SiLU-mul rows of this block as bf16 pairs with the layer's epoch
      if (tid < kRB / 2 * kMaxB) {
        const int r2 = tid / kMaxB, b = tid % kMaxB;
        if (2 * r2 < t.nrows && b < P.B && !dead) {
          const uint32_t pr = (uint32_t)f32_to_bf16_bits(S.hbuf[(2 * r2) * kMaxB + b]) |
                              ((uint32_t)f32_to_bf16_bits(S.hbuf[(2 * r2 + 1) * kMaxB + b]) << 16);
          st_word(P.hh + ((size_t)t.layer * P.B + b) * (P.ffn / 2) + (t.row0 + 2 * r2) / 2, pr,
                  epoch(t.layer, E_UP));
        }
      }
      consumer_sync();
    }
  }

  __device__ void emit(const Tile& t, int r, int b, float v) {
    const int row = t.row0 + r;
    const int qd = P.H * P.D, kd = P.Hkv * P.D;
    switch (t.kind) {
      case T_QKV: {
        const int off = t.seg == 0 ? row : (t.seg == 1 ? qd + row : qd + kd + row);
        st_word(P.qkv + ((size_t)t.layer * P.B + b) * (qd + 2 * kd) + off, __float_as_uint(v),
                epoch(t.layer, E_QKV));
        break;
      }
      case T_O:
      case T_DOWN: {
        float& xo = S.xown[b * kRB + r];
        xo += v;
        unsigned long long* buf = t.kind == T_O ? P.xo : P.xd;
        st_word(buf + ((size_t)t.layer * P.B + b) * P.hidden + row, __float_as_uint(xo),
                epoch(t.layer, t.kind == T_O ? E_O : E_DOWN));
        break;
      }
      case T_GATE:
        S.hbuf[r * kMaxB + b] = v;
        break;
      case T_UP: {
        const float z = S.hbuf[r * kMaxB + b];
        S.hbuf[r * kMaxB + b] = z / (1.0f + expf(-z)) * v;
        break;
      }
      case T_HEAD:
        P.logits[(size_t)b * P.vocab + row] = v;
        break;
    }
  }

  // ---- one stage (32 KV rows) of attention item (b, g, s). The first stage
  // loads and prepares the item's q heads (and the new k, v row when the
  // item holds position pos); every stage updates the running softmax of
  // thread (h, d); the last stage publishes the item's (o, max, sum).
  // Every consumer thread runs every barrier below; `live` only gates work.
  __device__ void attention(const Tile& t, uint8_t* stage, bool stage_ok) {
    const int l = t.layer, b = t.b, g = t.g, D = P.D, Gq = P.H / P.Hkv;
    const int qd = P.H * P.D, kd = P.Hkv * P.D;
    const int pos = si.L[b] - 1;
    const bool item_mine = pos >= t.s * kCHI && pos < (t.s + 1) * kCHI;
    const bool stage_mine = pos >= t.row0 && pos < t.row0 + t.nrows;
    uint16_t* Kc = reinterpret_cast<uint16_t*>(stage);
    uint16_t* Vc = reinterpret_cast<uint16_t*>(stage + kCH * kMaxD * 2);
    const int half = D >> 1;
    bool live;
    log(t.sub == 0 ? 1 : 3);
    if (t.sub == 0) {
      const unsigned long long* src = P.qkv + ((size_t)l * P.B + b) * (qd + 2 * kd);
      const unsigned ep = epoch(l, E_QKV);
      float* qs = S.qs;
      float* kv = S.kv;
      bool ok = stage_ok && !dead;
      ok = poll(src + g * Gq * D, Gq * D, ep, 0x800u,
                [&](int i, unsigned v) { qs[(i / D) * kMaxD + i % D] = __uint_as_float(v); }) && ok;
      if (item_mine) {
        ok = poll(src + qd + g * D, D, ep, 0x801u,
                  [&](int i, unsigned v) { kv[i] = __uint_as_float(v); }) && ok;
        ok = poll(src + qd + kd + g * D, D, ep, 0x802u,
                  [&](int i, unsigned v) { kv[kMaxD + i] = __uint_as_float(v); }) && ok;
      }
      live = all_ok(ok);
      log(2);
      hm = -INFINITY;
      hl = 0.f;
#pragma unroll
      for (int e = 0; e < kPer; ++e) ao[e] = 0.f;
      // per-head norm + RoPE: warp job = a q head (Gq of them), then k
      const int njobs = live ? Gq + (item_mine ? 1 : 0) : 0;
      const float* rope = S.rope + b * (kMaxD / 2) * 2;
      for (int job = warp; job < njobs; job += kCW) {
        const bool isq = job < Gq;
        float* hv = isq ? S.qs + job * kMaxD : S.kv;
        const uint16_t* nw = isq ? P.layer[l].q_norm : P.layer[l].k_norm;
        float x1[kMaxD / 64], x2[kMaxD / 64];
        float ss = 0.f;
#pragma unroll
        for (int j = 0; j < kMaxD / 64; ++j) {
          const int i = lane + 32 * j;
          x1[j] = i < half ? hv[i] : 0.f;
          x2[j] = i < half ? hv[i + half] : 0.f;
          ss = fmaf(x1[j], x1[j], fmaf(x2[j], x2[j], ss));
        }
        ss = warp_sum(ss);
        const float inv = 1.0f / sqrtf(ss / (float)D + P.eps);
#pragma unroll
        for (int j = 0; j < kMaxD / 64; ++j) {
          const int i = lane + 32 * j;
          if (i < half) {
            const float a = x1[j] * inv * bf16_bits_to_f32(__ldg(nw + i));
            const float c2 = x2[j] * inv * bf16_bits_to_f32(__ldg(nw + i + half));
            const float cs = rope[2 * i], sn = rope[2 * i + 1];
            const float r1 = a * cs - c2 * sn, r2 = c2 * cs + a * sn;
            hv[i] = isq ? r1 * P.scale : r1;
            hv[i + half] = isq ? r2 * P.scale : r2;
          }
        }
      }
      consumer_sync();
      if (live && item_mine) {
        // the new K (normed, rotated) and V rows, bf16, into the cache
        const size_t off = ((((size_t)l * P.B + b) * P.Hkv + g) * P.cap + pos) * D;
        for (int i = tid; i < 2 * D; i += kCT) {
          const uint16_t v = f32_to_bf16_bits(S.kv[(i / D) * kMaxD + i % D]);
          (i < D ? P.kc : P.vc)[off + i % D] = v;
        }
      }
    } else {
      live = stage_ok && !dead;  // per warp; the barriers below are unconditional
    }
    if (live && stage_mine) {  // this stage's copy of row pos predates its write
      for (int i = tid; i < 2 * D; i += kCT) {
        const uint16_t v = f32_to_bf16_bits(S.kv[(i / D) * kMaxD + i % D]);
        (i < D ? Kc : Vc)[(pos - t.row0) * D + i % D] = v;
      }
    }
    consumer_sync();
    // scores, warp h = query head h, lane r = row r; then the head's running
    // max, this stage's weights p_r = exp(s_r - max) and the rescale factor
    if (live && warp < Gq) {
      const int h = warp, r = lane;
      float sc = -INFINITY;
      if (r < t.nrows) {
        const uint16_t* kr = Kc + r * D;
        const float* qh = S.qs + h * kMaxD;
        float d = 0.f;
        for (int jj = 0; jj < D / 8; ++jj) {
          const int j = (jj + r) % (D / 8);  // rotate to spread banks
          const uint4 kv = *reinterpret_cast<const uint4*>(kr + 8 * j);
          const float4 qa = *reinterpret_cast<const float4*>(qh + 8 * j);
          const float4 qb = *reinterpret_cast<const float4*>(qh + 8 * j + 4);
          d = fmaf(qa.x, bf16_lo(kv.x), d); d = fmaf(qa.y, bf16_hi(kv.x), d);
          d = fmaf(qa.z, bf16_lo(kv.y), d); d = fmaf(qa.w, bf16_hi(kv.y), d);
          d = fmaf(qb.x, bf16_lo(kv.z), d); d = fmaf(qb.y, bf16_hi(kv.z), d);
          d = fmaf(qb.z, bf16_lo(kv.w), d); d = fmaf(qb.w, bf16_hi(kv.w), d);
        }
        sc = d;
      }
      const float m = fmaxf(hm, warp_max(sc));
      const float pr = r < t.nrows ? expf(sc - m) : 0.f;
      const float a = expf(hm - m);  // 0 on the first stage (hm = -inf)
      hl = fmaf(hl, a, warp_sum(pr));
      hm = m;
      S.sc[h * kCH + r] = pr;
      if (r == 0) S.sc[kMaxG * kCH + h] = a;
    }
    consumer_sync();
    // o = o * a_h + sum_r p_r v_r: thread element (h, d)
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      const int i = tid + e * kCT;
      if (!live || i >= Gq * D) continue;
      const int h = i / D, d = i % D;
      const float* ph = S.sc + h * kCH;
      float o = 0.f;
      for (int r = 0; r < t.nrows; ++r) o = fmaf(ph[r], bf16_bits_to_f32(Vc[r * D + d]), o);
      ao[e] = fmaf(ao[e], S.sc[kMaxG * kCH + h], o);
    }
    if (t.last && live) {
      const unsigned epa = epoch(l, E_ATT);
#pragma unroll
      for (int e = 0; e < kPer; ++e) {
        const int i = tid + e * kCT;
        if (i >= Gq * D) continue;
        const int h = i / D, d = i % D;
        st_word(P.part + ((((size_t)l * P.B + b) * P.H + g * Gq + h) * P.maxsplit + t.s) * (D + 2) + d,
                __float_as_uint(ao[e]), epa);
      }
      if (warp < Gq && lane == 0) {
        unsigned long long* pw =
            P.part + ((((size_t)l * P.B + b) * P.H + g * Gq + warp) * P.maxsplit + t.s) * (D + 2);
        st_word(pw + D, __float_as_uint(hm), epa);
        st_word(pw + D + 1, __float_as_uint(hl), epa);
      }
    }
    consumer_sync();
  }
};

__global__ void __launch_bounds__(kThreads, 1) decode_mega_kernel(const __grid_constant__ Params P) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + 32;
  int* flag = reinterpret_cast<int*>(smem + 512);
  uint8_t* p = smem + 1024;
  const int qd = P.H * P.D;
  const int Kmax = max(P.hidden, max(qd, P.ffn));
  Smem S;
  S.xs = Kmax + 8;
  S.gs = Kmax / 64;
  S.rope = reinterpret_cast<float*>(p);  p += kMaxB * kMaxD * 4;
  S.xown = reinterpret_cast<float*>(p);  p += kMaxB * kRB * 4;
  S.hbuf = reinterpret_cast<float*>(p);  p += kRB * kMaxB * 4;
  S.red = reinterpret_cast<float*>(p);   p += kCW * kRB * 8 * 4;
  S.qs = reinterpret_cast<float*>(p);    p += kMaxG * kMaxD * 4;
  S.kv = reinterpret_cast<float*>(p);    p += 2 * kMaxD * 4;
  S.sc = reinterpret_cast<float*>(p);    p += (kMaxG * kCH + kMaxG) * 4;
  S.ml = reinterpret_cast<float*>(p);    p += ((P.H * P.maxsplit * 2 * 4 + 127) / 128) * 128;
  S.bsc = reinterpret_cast<uint16_t*>(p); p += ((2 * kRB * (Kmax / 64) * 2 + 127) / 128) * 128;
  S.gsum = reinterpret_cast<float*>(p);  p += ((kMaxB * Kmax / 64 * 4 + 127) / 128) * 128;
  S.xstage = reinterpret_cast<float*>(p); p += ((kMaxB * P.hidden * 4 + 127) / 128) * 128;
  S.xin = reinterpret_cast<uint16_t*>(p); p += ((kMaxB * S.xs * 2 + 127) / 128) * 128;
  uint8_t* ring = reinterpret_cast<uint8_t*>(((uintptr_t)p + 1023) & ~(uintptr_t)1023);
  S.flag = flag;

  if (tid == 0) {
    for (int i = 0; i < P.stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kCW);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  SeqInfo si;
  seq_info(P, si);
  for (int i = tid; i < kMaxB * (P.D / 2); i += kThreads) {
    const int b = i / (P.D / 2), j = i % (P.D / 2);
    const int pos = si.L[b] > 0 ? si.L[b] - 1 : 0;
    const double inv_freq = pow(P.theta, -2.0 * (double)j / (double)P.D);
    double sd, cd;
    sincos((double)pos * inv_freq, &sd, &cd);
    S.rope[(b * (kMaxD / 2) + j) * 2] = (float)cd;
    S.rope[(b * (kMaxD / 2) + j) * 2 + 1] = (float)sd;
  }
  // every CTA reads the step counter before any CTA may advance it
  if (tid == 0) {
    flag[4] = (int)(*reinterpret_cast<volatile unsigned*>(P.step) * 512u + 1u);
    __threadfence();
    atomicAdd(P.cnt + C_START, 1u);
  }
  __syncthreads();
  const unsigned base = (unsigned)flag[4];

  if (warp == kCW) {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    Producer pr{P, ring, full, empty, pol, lane};
    walk(P, si, pr);
    pr.drain();
    return;
  }
  Consumer cs{P, si, S, ring, full, empty, base};
  cs.tid = tid;
  cs.warp = warp;
  cs.lane = lane;
  walk(P, si, cs);
  // advance the step counter (the next step's epochs) once every CTA has read it
  if (blockIdx.x == 0 && tid == 0) {
    const unsigned long long t0 = now_ns();
    while (ld_acquire(P.cnt + C_START) < gridDim.x && now_ns() - t0 < kWaitNs) {
    }
    atomicAdd(P.step, 1u);
  }
}

}  // namespace mk

// --------------------------------------------------------------- host ----

static size_t mega_smem_fixed(int hidden, int Kmax, int H, int maxsplit) {
  using namespace mk;
  size_t s = 1024;
  s += kMaxB * kMaxD * 4 + kMaxB * kRB * 4 + kRB * kMaxB * 4 + kCW * kRB * 8 * 4 +
       kMaxG * kMaxD * 4 + 2 * kMaxD * 4 + (kMaxG * kCH + kMaxG) * 4;
  s += ((size_t)(H * maxsplit * 2 * 4 + 127) / 128) * 128;
  s += ((size_t)(2 * kRB * (Kmax / 64) * 2 + 127) / 128) * 128;
  s += ((size_t)(kMaxB * Kmax / 64 * 4 + 127) / 128) * 128;
  s += ((size_t)(kMaxB * hidden * 4 + 127) / 128) * 128;
  s += ((size_t)(kMaxB * (Kmax + 8) * 2 + 127) / 128) * 128;
  return s + 1024;  // ring alignment slack
}

static size_t mega_stage_bytes(int Kmax) {
  return (size_t)mk::kStageW + 2 * mk::kRB * (Kmax / 64) * 2;
}

static const size_t kSmemBudget = 227 * 1024;

static int mega_maxsplit(int cap) { return (cap + mk::kCHI - 1) / mk::kCHI; }

bool mega_eligible(const qg_qwen3_config& c, int B, int cap) {
  using namespace mk;
  if (B < 1 || B > kMaxB) return false;
  if (c.layers < 1 || c.layers > kMaxLayers) return false;
  if (c.head_dim > kMaxD || c.head_dim % 64 != 0) return false;
  if (c.heads / c.kv_heads > kMaxG) return false;
  const int qd = c.heads * c.head_dim;
  for (int K : {c.hidden, qd, c.ffn})
    if (K % 512 != 0) return false;
  if ((c.kv_heads * c.head_dim) % kRB != 0) return false;
  if (c.heads * mega_maxsplit(cap) > 1024) return false;
  const int G = num_sms();
  if ((c.hidden / kRB + G - 1) / G > 1) return false;  // one residual block per CTA at most
  const int Kmax = std::max(c.hidden, std::max(qd, c.ffn));
  return mega_smem_fixed(c.hidden, Kmax, c.heads, mega_maxsplit(cap)) +
             4 * mega_stage_bytes(Kmax) <= kSmemBudget;
}

size_t mega_ws_bytes(const qg_qwen3_config& c, int B, int cap) {
  const size_t L = c.layers, qd = (size_t)c.heads * c.head_dim, kd = (size_t)c.kv_heads * c.head_dim;
  const size_t ms = (size_t)mega_maxsplit(cap);
  size_t words = 0;
  words += 2 * L * B * c.hidden;                     // xo, xd
  words += L * B * (qd + 2 * kd);                    // qkv
  words += L * B * c.heads * ms * (c.head_dim + 2);  // part
  words += L * B * c.ffn / 2;                        // hh
  return words * 8;
}

cudaError_t mega_launch(const qg_qwen3_config& c, const qg_qwen3_weights& w, uint16_t* kc,
                        uint16_t* vc, int cap, const int32_t* tokens, const int32_t* positions,
                        float* logits, int B, float* x, void* xws, unsigned* cnt, unsigned* step,
                        bool test_stall, unsigned long long* trace, cudaStream_t st) {
  using namespace mk;
  Params P;
  memset(&P, 0, sizeof(P));
  P.test_stall = test_stall ? 1 : 0;
  P.trace = trace;
  // the event log follows the phase stamps in the trace region
  P.log = trace ? trace + (size_t)num_sms() * (c.layers + 1) * 16 : nullptr;
  P.hidden = c.hidden; P.nlayers = c.layers; P.H = c.heads; P.Hkv = c.kv_heads; P.D = c.head_dim;
  P.ffn = c.ffn; P.vocab = c.vocab; P.B = B; P.cap = cap; P.eps = c.eps; P.theta = c.theta;
  P.scale = 1.0f / sqrtf((float)c.head_dim);
  P.maxsplit = mega_maxsplit(cap);
  P.ew = reinterpret_cast<const uint8_t*>(w.embed.w); P.es = w.embed.scales; P.eb = w.embed.biases;
  P.final_norm = w.final_norm;
  P.kc = kc; P.vc = vc; P.tokens = tokens; P.positions = positions; P.logits = logits;
  P.x = x; P.cnt = cnt; P.step = step;
  const size_t L = c.layers, qd = (size_t)c.heads * c.head_dim, kd = (size_t)c.kv_heads * c.head_dim;
  unsigned long long* wp = reinterpret_cast<unsigned long long*>(xws);
  P.xo = wp;   wp += L * B * c.hidden;
  P.xd = wp;   wp += L * B * c.hidden;
  P.qkv = wp;  wp += L * B * (qd + 2 * kd);
  P.part = wp; wp += L * B * c.heads * P.maxsplit * (c.head_dim + 2);
  P.hh = wp;
  for (int l = 0; l < c.layers; ++l) {
    const qg_qwen3_layer& Ly = w.layers[l];
    const qg_affine8_matrix* m[7] = {&Ly.q, &Ly.k, &Ly.v, &Ly.o, &Ly.gate, &Ly.up, &Ly.down};
    for (int i = 0; i < 7; ++i) {
      P.layer[l].w[i] = reinterpret_cast<const uint8_t*>(m[i]->w);
      P.layer[l].s[i] = m[i]->scales;
      P.layer[l].b[i] = m[i]->biases;
    }
    P.layer[l].in_norm = Ly.input_norm; P.layer[l].post_norm = Ly.post_norm;
    P.layer[l].q_norm = Ly.q_norm; P.layer[l].k_norm = Ly.k_norm;
  }
  const int Kmax = std::max(c.hidden, std::max(c.heads * c.head_dim, c.ffn));
  const size_t fixed = mega_smem_fixed(c.hidden, Kmax, c.heads, P.maxsplit);
  const size_t sbytes = mega_stage_bytes(Kmax);
  int stages = (int)((kSmemBudget - fixed) / sbytes);
  if (stages > 16) stages = 16;
  P.stages = stages;
  P.stage_bytes = (int)sbytes;
  const size_t smem = fixed + (size_t)stages * sbytes;
  static bool attr_done = false;
  if (!attr_done) {
    cudaFuncSetAttribute(decode_mega_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)kSmemBudget);
    attr_done = true;
  }
  cudaMemsetAsync(cnt, 0, 64, st);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(num_sms());
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  count_launch();
  return cudaLaunchKernelEx(&cfg, decode_mega_kernel, P);
}

}  // namespace qg
