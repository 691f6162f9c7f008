// Affine-INT8 group-64 matmul for a few activation rows (T <= 32) on the
// tcgen05 tensor cores (sm_100a): the batched LM head of a decode step.
//
//   Y[n][r] = sum_g ( s[r][g] * sum_{k in g} (q[r][k] - 128) x[n][k]
//                     + (beta[r][g] + 128 s[r][g]) * sum_{k in g} x[n][k] )  (+ R[n][r])
//
// the affine factorisation of w = q * s + beta over each group g of 64
// columns (turbospark-runtime 0.3.0, src/qwen3_asr_metal.rs, PackedLinear /
// load_packed_linear; the same arithmetic as the GEMV). The centred codes
// q - 128 lie in [-128, 127] and are exact in fp16, and so is x * 2^-e in
// fp16's normal range (x bf16, e a power-of-two prescale chosen from
// max|x| so that nothing overflows), so the MMA operands carry no
// dequantisation at all: the codes go to the tensor core as they are, and
// each group's scale and bias are applied to its partial sums afterwards.
//
// Persistent: one CTA per SM walks the 128-row tiles of W blockIdx.x,
// + gridDim.x, ..., each over all K, for NT = 16 or 32 rows of X. A stage is
// two groups (128 columns); a CTA's stages in order, tile after tile, run
// through one ring, so nothing drains between tiles. Roles of a CTA:
//   * the last warp (one lane) streams each stage's raw code bytes [128][128]
//     by TMA (128-byte swizzle) into a ring of shared-memory slots (those of
//     the first slots before the programmatic-dependent-launch wait);
//   * warps 0-7 (thread = row = tensor-memory lane; warp w: lane quadrant
//     w % 4, group w / 4) turn a stage's codes into fp16 pairs q - 128 (one
//     byte permute and one packed subtract per two codes) and store them
//     into tensor memory with tcgen05.st, where the MMA reads them as its A
//     operand;
//   * warp 12 owns tensor memory; its lane 0 issues, per group, four
//     tcgen05.mma (M = 128, N = NT, K = 16, A from tensor memory, B = X from
//     shared memory) into the group's accumulator;
//   * warps 8-11 (thread = row of the tile = tensor-memory lane) first form,
//     once per CTA from X in global memory, the sums of x per group and row
//     and max|x| (hence e), and write all of X as fp16 x * 2^-e in the K-major
//     128-byte swizzled layout the tensor core reads, where it stays for
//     every tile (NT K 2 <= 64 KB); then they drain each group's accumulator
//     with tcgen05.ld and fold it into fp32 registers with the group's scale
//     (times 2^e) and bias, and store each tile's Y (+ R).
// Tensor memory holds a ring of stage slots (5 at NT = 16, 4 at NT = 32):
// a code tile and an accumulator pair each, with one barrier pair per slot
// (filled: converters and drains; done: one MMA commit).
// Every wait is bounded (1 s); a wait that gives up sets a CTA-wide abort
// flag and the caller's error word, and tensor memory is freed only after
// the last commit has landed.
#include <cuda.h>

#include "qg_internal.cuh"
#include "tcgen05_util.cuh"

namespace qg {
namespace gas {

using namespace tc;

constexpr int kBM = 128;
constexpr int kBK = 64;                  // columns of a quantization group
constexpr int kMaxGroups = 32;           // K <= 2048 (scales kept in registers)
constexpr int kMaxSegs = 3;
constexpr int kConv = 8;                 // converter warps
constexpr int kThreads = 32 * (kConv + 6);  // converters, 4 drains, MMA, TMA
// A stage is two groups (128 columns of K): one TMA of codes, one round of
// waits and commits for two groups' MMAs. The converted codes live in
// tensor memory, as the MMA's A operand.
constexpr int kRing = 8;                   // stages of raw codes in flight
// stages in tensor memory (a code tile of two groups and an accumulator
// pair each): 5 at NT = 16 (160 + 320 of the 512 columns), 4 at NT = 32
constexpr int acc_slots(int NT) { return 2 * 5 * NT + 5 * 64 <= 512 ? 5 : 4; }
constexpr int kSlot = kBM * 2 * kBK;       // raw code bytes of two groups, 16 KB
constexpr int kXBytes = 64 * 1024;     // resident X: NT * K * 2 <= 64 KB
constexpr int kSmem = 1024 + kXBytes + kRing * kSlot + kMaxGroups * 32 * 4 +
                      2 * kMaxGroups * 128 * 2 + 512;

struct Seg {
  const uint16_t* s;   // bf16 [N][K/64]
  const uint16_t* b;   // bf16 [N][K/64]
  void* y;             // [T][N] fp32 or bf16
  const float* res;    // fp32 [T][N] or null
  int N;
  int y_bf16;
  int tile0;           // first 128-row tile of this segment in the launch
};

struct Params {
  Seg seg[kMaxSegs];
  int nseg, T, K;
  const uint16_t* x;   // bf16 [T][K] (for the per-group sums)
};

struct Maps {
  CUtensorMap w[kMaxSegs];  // codes u8 [N][K] in boxes of 64 x 128
};

__device__ __forceinline__ int seg_of(const Params& P, int tile) {
  int si = 0;
#pragma unroll
  for (int i = 1; i < kMaxSegs; ++i)
    if (i < P.nseg && tile >= P.seg[i].tile0) si = i;
  return si;
}

template <int NT>
__device__ __forceinline__ void tmem_ld(uint32_t ta, uint32_t (&v)[NT]);
template <>
__device__ __forceinline__ void tmem_ld<16>(uint32_t ta, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15])
      : "r"(ta));
}
template <>
__device__ __forceinline__ void tmem_ld<32>(uint32_t ta, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]),
        "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]),
        "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(ta));
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

template <int NT>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_affine8_skinny_kernel(const __grid_constant__ Maps maps, const __grid_constant__ Params P,
                               int tiles, unsigned* __restrict__ err) {
  // tensor memory: kAcc accumulator pairs (2 NT columns each), then the ring
  // of converted code tiles (two groups of 32 columns each). Stage j uses
  // pair and tile j % kAcc; one barrier pair per slot serves both:
  // ready[b] completes when the converters have filled the tile and the
  // drains have read the pair's previous accumulators, done[b] (one commit)
  // when the stage's MMAs are done.
  constexpr int kAcc = acc_slots(NT);
  constexpr int kAccCols = 2 * kAcc * NT;
  static_assert(kAccCols + kAcc * 64 <= 512, "tensor memory");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* xres = smem;                           // [K/64][NT][64] fp16, swizzled
  uint8_t* slots = smem + kXBytes;                // [kRing][128][128] raw codes, swizzled
  float* sx = reinterpret_cast<float*>(slots + kRing * kSlot);  // [K/64][NT]
  uint16_t* tsc = reinterpret_cast<uint16_t*>(sx + kMaxGroups * 32);  // [K/64][128] scales
  uint16_t* tbi = tsc + kMaxGroups * 128;                             // [K/64][128] biases
  uint64_t* r_raw = reinterpret_cast<uint64_t*>(tbi + kMaxGroups * 128);  // codes landed
  uint64_t* r_free = r_raw + kRing;               // codes read by the converters
  uint64_t* ready = r_free + kRing;               // [kAcc] tile converted, pair free
  uint64_t* done = ready + kAcc;                  // [kAcc] the stage's MMAs done
  uint64_t* xready = done + kAcc;                 // X resident (fp16, swizzled)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(xready + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int K = P.K, nk = K / kBK, ns = nk / 2;  // groups, stages (two groups each) per tile
  // this CTA's tiles: blockIdx.x, + gridDim.x, ...; their stages in order,
  // tile after tile, are the stages j = i * ns + ks of one ring
  const int ntl = ((int)blockIdx.x < tiles) ? (tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  const int total = ntl * ns;

  if (tid == 0) {
    for (int s = 0; s < kRing; ++s) {
      mbar_init(&r_raw[s], 1);
      mbar_init(&r_free[s], 32 * kConv);
    }
    for (int b = 0; b < kAcc; ++b) {
      mbar_init(&ready[b], 32 * kConv + 128);  // the converters and the drains
      mbar_init(&done[b], 1);
    }
    mbar_init(xready, 128);
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kConv + 4) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;
  // the next kernel of a chain may start its own weight loads
  pdl_trigger();

  bool ok = true;
  if (warp == kConv + 5) {
    // ------------------------------------------------------------ TMA
    if (lane == 0) {
      auto load_codes = [&](int j, int s) {
        const int tile = (int)blockIdx.x + (j / ns) * (int)gridDim.x, ks = j % ns;
        const int si = seg_of(P, tile);
        const int row0 = (tile - P.seg[si].tile0) * kBM;
        mbar_expect_tx(&r_raw[s], (uint32_t)kSlot);
        tma_load_2d(smem_u32(slots + (size_t)s * kSlot), &maps.w[si], ks * 2 * kBK, row0,
                    &r_raw[s]);
      };
      // weights never depend on the previous kernel: no wait here
      const int pre = total < kRing ? total : kRing;
      for (int j = 0; j < pre; ++j) load_codes(j, j);
      int issued = pre;
      for (int j = pre; j < total; ++j) {
        const int s = j % kRing;
        if (!wait_bar(&r_free[s], (uint32_t)((j / kRing) + 1) & 1u, abort)) {
          ok = false;
          *abort = 1;
          break;
        }
        load_codes(j, s);
        ++issued;
      }
      // no copy may land after the CTA is gone: wait (bounded) for the last
      // fill of every slot used
      for (int j = issued - kRing > 0 ? issued - kRing : 0; j < issued; ++j) {
        const int s = j % kRing;
        const uint32_t par = (uint32_t)(j / kRing) & 1u;
        if (!mbar_try_wait(&r_raw[s], par)) {
          const unsigned long long t0 = now_ns();
          while (!mbar_try_wait(&r_raw[s], par))
            if (now_ns() - t0 > kWaitNs) break;
        }
      }
    }
  } else if (warp < kConv) {
    // ------------------------------------------------------ converters
    // warp w: rows 32 (w % 4) + lane (its tensor-memory lanes) of group
    // w / 4 of each stage; a thread converts its row's 64 codes and stores
    // them with one tcgen05.st (32 columns of fp16 pairs)
    const int q = warp & 3, h = warp >> 2;
    const int r = 32 * q + lane;
    for (int j = 0; j < total; ++j) {
      const int s = j % kRing, a = j % kAcc;
      const uint32_t par = (uint32_t)(j / kRing) & 1u;
      if (!wait_bar(&r_raw[s], par, abort) ||
          (j >= kAcc && !wait_bar(&done[a], (uint32_t)((j / kAcc) + 1) & 1u, abort))) {
        ok = false;
        *abort = 1;
        break;
      }
      const uint8_t* row = slots + (size_t)s * kSlot + r * 128;
      uint32_t v[32];
#pragma unroll
      for (int c = 0; c < 4; ++c) {  // 16-byte chunk 4 h + c of the row, swizzled by TMA
        const uint4 w = *reinterpret_cast<const uint4*>(row + (((4 * h + c) ^ (r & 7)) << 4));
        v[8 * c + 0] = codes01(w.x);
        v[8 * c + 1] = codes23(w.x);
        v[8 * c + 2] = codes01(w.y);
        v[8 * c + 3] = codes23(w.y);
        v[8 * c + 4] = codes01(w.z);
        v[8 * c + 5] = codes23(w.z);
        v[8 * c + 6] = codes01(w.w);
        v[8 * c + 7] = codes23(w.w);
      }
      const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(kAccCols + a * 64 + h * 32);
      asm volatile(
          "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
          "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(ta),
          "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
          "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
          "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
          "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
          "r"(v[29]), "r"(v[30]), "r"(v[31])
          : "memory");
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      // the slot's raw codes are consumed only here: the store above used
      // every value loaded from it (arriving earlier would let the next TMA
      // overwrite the slot under loads still in flight)
      mbar_arrive(&r_free[s]);
      mbar_arrive(&ready[a]);
    }
    if (!ok) *abort = 1;
  } else if (warp == kConv + 4) {
    // ------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = instr_desc_f16<NT>();
      if (total > 0 && !wait_bar(xready, 0u, abort)) {
        ok = false;
        *abort = 1;
      }
      for (int j = 0; j < total && ok; ++j) {
        const int a = j % kAcc, b = a;
        if (!wait_bar(&ready[b], (uint32_t)(j / kAcc) & 1u, abort)) {
          ok = false;
          *abort = 1;
          break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const int g0 = (j % ns) * 2;  // the stage's first group
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const uint32_t ta = tmem + (uint32_t)(kAccCols + a * 64 + hh * 32);
          const uint32_t sb = smem_u32(xres + (size_t)(g0 + hh) * (NT * kBK * 2));
          const uint32_t d = tmem + (uint32_t)((2 * b + hh) * NT);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            const uint64_t db = smem_desc(sb + k * 32);
            const uint32_t acc = k > 0 ? 1u : 0u;
            asm volatile(
                "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
                " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d),
                "r"(ta + (uint32_t)(k * 8)), "l"(db), "r"(idesc), "r"(acc)
                : "memory");
          }
        }
        asm volatile(
            "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                smem_u32(&done[b]))
            : "memory");
      }
    }
  } else {
    // --------------------------------------------------------- drains
    const int q = warp & 3;  // tensor-memory lanes 32 q .. 32 q + 31
    const int Kg = K / 64;
    const int col = tid - 32 * kConv;  // this drain thread's row of the tile
    // the sum of each group of x per row (rows past T are zero), in order:
    // X is the same for every tile, so once per CTA
    // every accumulator pair starts free
    for (int b = 0; b < kAcc; ++b) mbar_arrive(&ready[b]);
    pdl_wait();  // x is written by the previous kernel
    float mx = 0.f;
    for (int i = col; i < Kg * NT; i += 128) {
      const int g = i / NT, n = i % NT;
      float a = 0.f;
      if (n < P.T) {
        const uint4* xp = reinterpret_cast<const uint4*>(P.x + (size_t)n * K + g * 64);
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const uint4 v = __ldcg(xp + jj);
          const float f[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                              bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
          a += ((f[0] + f[1]) + (f[2] + f[3])) + ((f[4] + f[5]) + (f[6] + f[7]));
#pragma unroll
          for (int e = 0; e < 8; ++e) mx = fmaxf(mx, fabsf(f[e]));
        }
      }
      sx[i] = a;
    }
    // the prescale 2^-e: max|x| * 2^-e < 2^15 (NaN or inf in x propagate
    // to y without one)
    mx = warp_max(mx);
    float* red = reinterpret_cast<float*>(tsc);  // scratch until the first tile's scales
    if (lane == 0) red[q] = mx;
    asm volatile("bar.sync 1, 128;" ::: "memory");
    mx = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    const int e = (mx >= 32768.f && mx <= 3.0e38f) ? (int)ceilf(log2f(mx / 16384.f)) : 0;
    const float up = exp2f((float)e);
    asm volatile("bar.sync 1, 128;" ::: "memory");  // red is read by all before reuse
    // all of X as fp16 x * 2^-e, group g's [NT][64] tile at g * NT * 128
    // bytes, 16-byte chunk c of row n at chunk c ^ (n % 8) (rows past T zero)
    const float down = exp2f((float)-e);
    for (int i = col; i < Kg * NT * 8; i += 128) {
      const int g = i / (NT * 8), n = (i / 8) % NT, c = i % 8;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (n < P.T) {
        const uint4 xv = __ldcg(reinterpret_cast<const uint4*>(P.x + (size_t)n * K + g * 64 + c * 8));
        const uint32_t w4[4] = {xv.x, xv.y, xv.z, xv.w};
        uint32_t h4[4];
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2) {
          const __half2 h = __floats2half2_rn(bf16_lo(w4[e2]) * down, bf16_hi(w4[e2]) * down);
          h4[e2] = *reinterpret_cast<const uint32_t*>(&h);
        }
        v = make_uint4(h4[0], h4[1], h4[2], h4[3]);
      }
      *reinterpret_cast<uint4*>(xres + (size_t)g * NT * 128 + n * 128 + ((c ^ (n & 7)) << 4)) = v;
    }
    // make the generic-proxy stores visible to the tensor core
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    mbar_arrive(xready);
    // per tile: this row's bf16 scale and bias per group in its own column
    // of tsc / tbi; the fp32 accumulators of the NT rows
    float acc[NT];
    int r = 0;
    const Seg* Sg = &P.seg[0];
    for (int j = 0; j < total; ++j) {
      const int ks = j % ns, b = j % kAcc;
      if (ks == 0) {
        const int tile = (int)blockIdx.x + (j / ns) * (int)gridDim.x;
        Sg = &P.seg[seg_of(P, tile)];
        r = (tile - Sg->tile0) * kBM + 32 * q + lane;  // rows past N are never stored
        const int rc = min(r, Sg->N - 1);
        for (int g = 0; g < Kg; ++g) {
          tsc[g * 128 + col] = __ldg(Sg->s + (size_t)rc * Kg + g);
          tbi[g * 128 + col] = __ldg(Sg->b + (size_t)rc * Kg + g);
        }
#pragma unroll
        for (int n = 0; n < NT; ++n) acc[n] = 0.f;
      }
      if (!wait_bar(&done[b], (uint32_t)(j / kAcc) & 1u, abort)) {
        ok = false;
        *abort = 1;
        break;
      }
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      uint32_t v0[NT], v1[NT];
      tmem_ld<NT>(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(2 * b * NT), v0);
      tmem_ld<NT>(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)((2 * b + 1) * NT), v1);
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      mbar_arrive(&ready[b]);  // the pair is free for stage j + kAcc
      const int g0 = 2 * ks;
      const float s0 = bf16_bits_to_f32(tsc[g0 * 128 + col]);
      const float s1 = bf16_bits_to_f32(tsc[(g0 + 1) * 128 + col]);
      const float c0 = fmaf(128.f, s0, bf16_bits_to_f32(tbi[g0 * 128 + col]));
      const float c1 = fmaf(128.f, s1, bf16_bits_to_f32(tbi[(g0 + 1) * 128 + col]));
      const float u0 = s0 * up, u1 = s1 * up;
      const float* sx0 = sx + g0 * NT;
      const float* sx1 = sx0 + NT;
#pragma unroll
      for (int n = 0; n < NT; ++n)
        acc[n] = fmaf(u1, __uint_as_float(v1[n]),
                      fmaf(c1, sx1[n], fmaf(u0, __uint_as_float(v0[n]), fmaf(c0, sx0[n], acc[n]))));
      if (ks == ns - 1 && r < Sg->N) {
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          if (n >= P.T) break;
          const size_t o = (size_t)n * Sg->N + r;
          float val = acc[n];
          if (Sg->res) val += Sg->res[o];
          if (Sg->y_bf16)
            reinterpret_cast<uint16_t*>(Sg->y)[o] = f32_to_bf16_bits(val);
          else
            reinterpret_cast<float*>(Sg->y)[o] = val;
        }
      }
    }
    if (*abort) ok = false;
  }
  if (!ok && err) atomicOr(err, 1u);
  // every MMA has landed before tensor memory goes: the drains consumed the
  // last accumulator (or gave up, in which case the issuer also stopped)
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == kConv + 4) {
    __syncwarp();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

}  // namespace gas

// Whether the skinny matmul takes the launch: T <= 32 rows of X, K a
// multiple of 128 up to 2048, and X resident in shared memory as fp16 (its
// NT = 16 or 32 rows times K times 2 bytes within 64 KB).
bool gemm_affine8_skinny_ok(int T, int K) {
  const int NT = T <= 16 ? 16 : 32;
  return T >= 1 && T <= 32 && K % 128 == 0 && K <= 2048 && NT * K * 2 <= 64 * 1024;
}

template <int NT>
static cudaError_t gas_launch(const gas::Maps& maps, const gas::Params& P, int tiles,
                              unsigned* err, cudaStream_t st, bool pdl) {
  ensure_smem((const void*)gas::gemm_affine8_skinny_kernel<NT>, gas::kSmem);
  // persistent: one CTA per SM walks its tiles
  const int grid = tiles < num_sms() ? tiles : num_sms();
  return launch_pdl(gas::gemm_affine8_skinny_kernel<NT>, dim3(grid), dim3(gas::kThreads),
                    (size_t)gas::kSmem, st, pdl, maps, P, tiles, err);
}

cudaError_t gemm_affine8_skinny_launch(const A8Seg* segs, int nseg, const uint16_t* X, int T,
                                       int K, unsigned* err, cudaStream_t st, bool pdl) {
  if (nseg < 1 || nseg > gas::kMaxSegs || !gemm_affine8_skinny_ok(T, K))
    return cudaErrorInvalidValue;
  gas::Params P = {};
  gas::Maps maps = {};
  P.nseg = nseg;
  P.T = T;
  P.K = K;
  P.x = X;
  int tiles = 0;
  for (int i = 0; i < nseg; ++i) {
    P.seg[i] = gas::Seg{segs[i].s, segs[i].b, segs[i].y, segs[i].res, segs[i].N, segs[i].y_bf16,
                        tiles};
    if (!make_u8_map(&maps.w[i], segs[i].w, segs[i].N, K, 2 * gas::kBK, gas::kBM, true))
      return cudaErrorInvalidValue;
    tiles += (segs[i].N + gas::kBM - 1) / gas::kBM;
  }
  if (tiles == 0) return cudaSuccess;
  if (T <= 16) return gas_launch<16>(maps, P, tiles, err, st, pdl);
  return gas_launch<32>(maps, P, tiles, err, st, pdl);
}

}  // namespace qg
