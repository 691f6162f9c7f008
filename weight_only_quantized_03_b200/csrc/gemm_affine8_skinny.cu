// Affine-INT8 group-64 matmul for a few activation rows (T <= 32) on the
// tcgen05 tensor cores (sm_100a): the batched LM head of a decode step.
//
//   Y[n][r] = sum_g ( s[r][g] * sum_{k in g} (q[r][k] - 128) x[n][k]
//                     + (beta[r][g] + 128 s[r][g]) * sum_{k in g} x[n][k] )  (+ R[n][r])
//
// the affine factorisation of w = q * s + beta over each group g of 64
// columns (turbospark-runtime 0.3.0, src/qwen3_asr_metal.rs, PackedLinear /
// load_packed_linear; the same arithmetic as the GEMV). The centred codes
// q - 128 lie in [-128, 127] and are exact in bf16, and so are their
// products with the bf16 activations in fp32, so the MMA operands carry no
// dequantisation at all: the codes go to the tensor core as they are, and
// each group's scale and bias are applied to its partial sums afterwards.
//
// Persistent: one CTA per SM walks the 128-row tiles of W blockIdx.x,
// + gridDim.x, ..., each over all K, for NT = 16 or 32 rows of X; its groups
// in order, tile after tile, are the stages of one ring, so nothing drains
// between tiles. Roles of a CTA:
//   * warp 9 (one lane) streams each group's raw code bytes [128][64] and
//     X's [NT][64] tile by TMA into a ring of stages (the codes of the first
//     stages before the programmatic-dependent-launch wait);
//   * warps 0-3 turn the codes into bf16 (q - 128) in the K-major 128-byte
//     swizzled layout the tensor core reads (16-byte chunk c of row r at
//     chunk c ^ (r % 8)): one byte permute and one add per code, one packing
//     permute per two;
//   * warp 8 owns tensor memory; its lane 0 issues, per group, four
//     tcgen05.mma (M = 128, N = NT, K = 16) into one of four accumulators
//     (groups take them in turn), commits the stage back to the ring and the
//     accumulator to the drain;
//   * warps 4-7 (thread = row of the tile = tensor-memory lane) drain each
//     group's accumulator with tcgen05.ld and fold it into fp32 registers
//     with the group's scale and bias (the sums of x per group and row are
//     formed once, from X in global memory), and store each tile's Y (+ R).
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
constexpr int kBK = 64;                  // one quantization group per stage
constexpr int kMaxGroups = 32;           // K <= 2048 (scales kept in registers)
constexpr int kMaxSegs = 3;
constexpr int kThreads = 320;            // 0-3 convert, 4-7 drain, 8 MMA, 9 TMA
constexpr int kStages = 6;
constexpr int kAcc = 4;                // accumulators in tensor memory (groups in flight)
constexpr int kStageA = kBM * kBK * 2;   // bf16 codes, 16 KB
constexpr int kStageX = 32 * kBK * 2;    // room for NT <= 32 rows of X
constexpr int kStageRaw = kBM * kBK;     // raw code bytes, 8 KB
constexpr int kStage = kStageA + kStageX + kStageRaw;  // 28 KB, a multiple of 1024
constexpr int kSmem = 1024 + kStages * kStage + kMaxGroups * 32 * 4 + 512;

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

// two codes (bytes j0, j0 + 1 of w) as a bf16 pair (q - 128): 2^23 + q in
// fp32 minus 2^23 + 128 is exact, and its upper half is the exact bf16
__device__ __forceinline__ uint32_t codes_bf16(uint32_t w, int j0) {
  const float f0 = __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7540u + j0)) - 8388736.0f;
  const float f1 = __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7541u + j0)) - 8388736.0f;
  return __byte_perm(__float_as_uint(f0), __float_as_uint(f1), 0x7632u);
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
    gemm_affine8_skinny_kernel(const __grid_constant__ CUtensorMap tmX,
                               const __grid_constant__ Maps maps, const __grid_constant__ Params P,
                               int tiles, unsigned* __restrict__ err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* stages = smem;
  float* sx = reinterpret_cast<float*>(smem + kStages * kStage);  // [K/64][NT]
  uint64_t* full_raw = reinterpret_cast<uint64_t*>(sx + kMaxGroups * 32);  // codes landed
  uint64_t* full_x = full_raw + kStages;                                     // X landed
  uint64_t* full_a = full_x + kStages;                                       // codes converted
  uint64_t* empty = full_a + kStages;
  uint64_t* acc_full = empty + kStages;     // [kAcc]
  uint64_t* acc_empty = acc_full + kAcc;    // [kAcc]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + kAcc);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int K = P.K, nk = K / kBK;
  // this CTA's tiles: blockIdx.x, + gridDim.x, ...; its groups in order,
  // tile after tile, are the stages j = i * nk + kb of one ring
  const int ntl = ((int)blockIdx.x < tiles) ? (tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  const int total = ntl * nk;
  constexpr uint32_t kTmemCols = kAcc * NT < 32 ? 32 : kAcc * NT;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_raw[s], 1);
      mbar_init(&full_x[s], 1);
      mbar_init(&full_a[s], 128);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < kAcc; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 8) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;
  // the next kernel of a chain may start its own weight loads
  pdl_trigger();

  bool ok = true;
  if (warp == 9) {
    // ------------------------------------------------------------ TMA
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmX)) : "memory");
      auto load_codes = [&](int j, int s) {
        const int tile = (int)blockIdx.x + (j / nk) * (int)gridDim.x, kb = j % nk;
        const int si = seg_of(P, tile);
        const int row0 = (tile - P.seg[si].tile0) * kBM;
        mbar_expect_tx(&full_raw[s], (uint32_t)kStageRaw);
        tma_load_2d(smem_u32(stages + (size_t)s * kStage + kStageA + kStageX), &maps.w[si],
                    kb * kBK, row0, &full_raw[s]);
      };
      auto load_x = [&](int j, int s) {
        mbar_expect_tx(&full_x[s], (uint32_t)(NT * kBK * 2));
        tma_load_2d(smem_u32(stages + (size_t)s * kStage + kStageA), &tmX, (j % nk) * kBK, 0,
                    &full_x[s]);
      };
      // the codes of the first stages go out before the wait (weights never
      // depend on the previous kernel), X's tiles after it
      const int pre = total < kStages ? total : kStages;
      for (int j = 0; j < pre; ++j) load_codes(j, j);
      pdl_wait();  // X is written by the previous kernel
      for (int j = 0; j < pre; ++j) load_x(j, j);
      int issued = pre;
      for (int j = pre; j < total; ++j) {
        const int s = j % kStages;
        if (!wait_bar(&empty[s], (uint32_t)((j / kStages) + 1) & 1u, abort)) {
          ok = false;
          *abort = 1;
          break;
        }
        load_codes(j, s);
        load_x(j, s);
        ++issued;
      }
      // no copy may land after the CTA is gone: wait (bounded) for the last
      // fill of every stage used
      for (int j = issued - kStages > 0 ? issued - kStages : 0; j < issued; ++j) {
        const int s = j % kStages;
        const uint32_t par = (uint32_t)(j / kStages) & 1u;
        for (uint64_t* bar : {&full_raw[s], &full_x[s]}) {
          if (!mbar_try_wait(bar, par)) {
            const unsigned long long t0 = now_ns();
            while (!mbar_try_wait(bar, par))
              if (now_ns() - t0 > kWaitNs) break;
          }
        }
      }
    }
  } else if (warp < 4) {
    // ------------------------------------------------------ converters
    for (int j = 0; j < total; ++j) {
      const int s = j % kStages;
      if (!wait_bar(&full_raw[s], (uint32_t)(j / kStages) & 1u, abort)) {
        ok = false;
        *abort = 1;
        break;
      }
      uint8_t* st = stages + (size_t)s * kStage;
      const uint8_t* raw = st + kStageA + kStageX;
#pragma unroll
      for (int it = 0; it < 4; ++it) {
        const int flat = it * 128 + tid;  // 16-byte piece: row flat / 4, columns 16 (flat % 4) ..
        const int r = flat >> 2, p = flat & 3;
        const uint4 c = *reinterpret_cast<const uint4*>(raw + r * kBK + p * 16);
        const uint4 lo = make_uint4(codes_bf16(c.x, 0), codes_bf16(c.x, 2), codes_bf16(c.y, 0),
                                    codes_bf16(c.y, 2));
        const uint4 hi = make_uint4(codes_bf16(c.z, 0), codes_bf16(c.z, 2), codes_bf16(c.w, 0),
                                    codes_bf16(c.w, 2));
        const int c0 = 2 * p;
        *reinterpret_cast<uint4*>(st + r * 128 + ((c0 ^ (r & 7)) << 4)) = lo;
        *reinterpret_cast<uint4*>(st + r * 128 + (((c0 + 1) ^ (r & 7)) << 4)) = hi;
      }
      // make the generic-proxy stores visible to the tensor core
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(&full_a[s]);
    }
    if (!ok) *abort = 1;
  } else if (warp == 8) {
    // ------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = instr_desc<NT>();
      for (int j = 0; j < total; ++j) {
        const int s = j % kStages, b = j % kAcc;
        const uint32_t par = (uint32_t)(j / kStages) & 1u;
        if (!wait_bar(&full_x[s], par, abort) || !wait_bar(&full_a[s], par, abort) ||
            (j >= kAcc && !wait_bar(&acc_empty[b], (uint32_t)((j / kAcc) + 1) & 1u, abort))) {
          ok = false;
          *abort = 1;
          break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t sa = smem_u32(stages + (size_t)s * kStage);
        const uint32_t sb = sa + kStageA;
        const uint32_t d = tmem + (uint32_t)(b * NT);
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k) {
          const uint64_t da = smem_desc(sa + k * 32), db = smem_desc(sb + k * 32);
          const uint32_t acc = k > 0 ? 1u : 0u;
          asm volatile(
              "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
              " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d),
              "l"(da), "l"(db), "r"(idesc), "r"(acc)
              : "memory");
        }
        asm volatile(
            "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                smem_u32(&empty[s]))
            : "memory");
        asm volatile(
            "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                smem_u32(&acc_full[b]))
            : "memory");
      }
    }
  } else {
    // --------------------------------------------------------- drains
    const int q = warp & 3;  // tensor-memory lanes 32 q .. 32 q + 31
    const int Kg = K / 64;
    // the sum of each group of x per row (rows past T are zero), in order:
    // X is the same for every tile, so once per CTA
    pdl_wait();  // x is written by the previous kernel
    for (int i = tid - 128; i < Kg * NT; i += 128) {
      const int g = i / NT, n = i % NT;
      float a = 0.f;
      if (n < P.T) {
        const uint4* xp = reinterpret_cast<const uint4*>(P.x + (size_t)n * K + g * 64);
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const uint4 v = __ldcg(xp + jj);
          a += ((bf16_lo(v.x) + bf16_hi(v.x)) + (bf16_lo(v.y) + bf16_hi(v.y))) +
               ((bf16_lo(v.z) + bf16_hi(v.z)) + (bf16_lo(v.w) + bf16_hi(v.w)));
        }
      }
      sx[i] = a;
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    // per tile: this row's scales and biases as bf16 pairs (group 2 m in
    // the low half of word m), the fp32 accumulators of the NT rows of X
    uint32_t sp[kMaxGroups / 2], bp[kMaxGroups / 2];
    float acc[NT];
    int r = 0;
    const Seg* Sg = &P.seg[0];
    for (int j = 0; j < total; ++j) {
      const int kb = j % nk, b = j % kAcc;
      if (kb == 0) {
        const int tile = (int)blockIdx.x + (j / nk) * (int)gridDim.x;
        Sg = &P.seg[seg_of(P, tile)];
        r = (tile - Sg->tile0) * kBM + 32 * q + lane;  // rows past N are never stored
        const int rc = min(r, Sg->N - 1);
#pragma unroll
        for (int m = 0; m < kMaxGroups / 2; ++m) {
          sp[m] = bp[m] = 0u;
          if (2 * m < Kg) {
            const uint16_t* s2 = Sg->s + (size_t)rc * Kg + 2 * m;
            const uint16_t* b2 = Sg->b + (size_t)rc * Kg + 2 * m;
            sp[m] = (uint32_t)__ldg(s2) | (2 * m + 1 < Kg ? (uint32_t)__ldg(s2 + 1) << 16 : 0u);
            bp[m] = (uint32_t)__ldg(b2) | (2 * m + 1 < Kg ? (uint32_t)__ldg(b2 + 1) << 16 : 0u);
          }
        }
#pragma unroll
        for (int n = 0; n < NT; ++n) acc[n] = 0.f;
      }
      if (!wait_bar(&acc_full[b], (uint32_t)(j / kAcc) & 1u, abort)) {
        ok = false;
        *abort = 1;
        break;
      }
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      uint32_t v[NT];
      tmem_ld<NT>(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * NT), v);
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      mbar_arrive(&acc_empty[b]);
      uint32_t s2 = 0u, b2 = 0u;
#pragma unroll
      for (int m = 0; m < kMaxGroups / 2; ++m)
        if (m == (kb >> 1)) {
          s2 = sp[m];
          b2 = bp[m];
        }
      const float s = (kb & 1) ? bf16_hi(s2) : bf16_lo(s2);
      const float c = fmaf(128.f, s, (kb & 1) ? bf16_hi(b2) : bf16_lo(b2));
      const float* sxg = sx + kb * NT;
#pragma unroll
      for (int n = 0; n < NT; ++n) acc[n] = fmaf(s, __uint_as_float(v[n]), fmaf(c, sxg[n], acc[n]));
      if (kb == nk - 1 && r < Sg->N) {
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
  if (warp == 8) {
    __syncwarp();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols));
  }
}

}  // namespace gas

// Whether the skinny matmul takes the launch: T <= 32 rows of X and K a
// multiple of 64 up to 2048 (the groups' scales stay in registers).
bool gemm_affine8_skinny_ok(int T, int K) { return T >= 1 && T <= 32 && K % 64 == 0 && K <= 2048; }

template <int NT>
static cudaError_t gas_launch(const CUtensorMap& tmX, const gas::Maps& maps, const gas::Params& P,
                              int tiles, unsigned* err, cudaStream_t st, bool pdl) {
  ensure_smem((const void*)gas::gemm_affine8_skinny_kernel<NT>, gas::kSmem);
  // persistent: one CTA per SM walks its tiles
  const int grid = tiles < num_sms() ? tiles : num_sms();
  return launch_pdl(gas::gemm_affine8_skinny_kernel<NT>, dim3(grid), dim3(gas::kThreads),
                    (size_t)gas::kSmem, st, pdl, tmX, maps, P, tiles, err);
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
    if (!make_u8_map(&maps.w[i], segs[i].w, segs[i].N, K, gas::kBK, gas::kBM))
      return cudaErrorInvalidValue;
    tiles += (segs[i].N + gas::kBM - 1) / gas::kBM;
  }
  if (tiles == 0) return cudaSuccess;
  const int NT = T <= 16 ? 16 : 32;
  CUtensorMap tmX;
  if (!make_bf16_map(&tmX, X, T, K, NT)) return cudaErrorInvalidValue;
  if (NT == 16) return gas_launch<16>(tmX, maps, P, tiles, err, st, pdl);
  return gas_launch<32>(tmX, maps, P, tiles, err, st, pdl);
}

}  // namespace qg
