// Q4_0 matmul on the tcgen05 tensor cores (sm_100a):
//
//   C[m][r] = sum_k bf16(A[m][k]) * bf16(d * (n - 8))[r][k]  (+ bias[r])
//
// Definition: fuel-transformers 0.19.1, src/models/lazy_quantized_whisper.rs,
// `q_linear` (y = x W^T + b with W held as GGUF Q4_0 blocks of 32: an fp16
// scale d then 16 bytes, byte j = code j | code j+16 << 4, w = d (n - 8)),
// applied by `encoder_layer` to all frames at once (M = frames). Operands are
// rounded to bf16 (nearest even) and multiplied with fp32 accumulation.
//
// Structure
//   1. a_to_bf16_kernel: A fp32 -> bf16 into the workspace (once per call;
//      every N tile then reads half the bytes).
//   2. K % 256 == 0 (every Whisper projection): gemm_q4_0_t_kernel, the
//      transposed form described at its definition (W dequantized into
//      tensor memory as the MMA's A operand, A's rows as its B operand).
//      Otherwise gemm_q4_0_tc_kernel, one CTA per 128 x BN output tile, over a ring of
//      shared-memory stages of 64 columns of K, both operands in the K-major
//      128-byte-swizzled layout the tensor core reads (16-byte chunk c of
//      row r at chunk c ^ (r % 8) of its 1024-byte atom):
//      * warp 9 loads A's 128 x 64 tile of each stage with one TMA tensor
//        copy (the 128-byte swizzle is the copy's own), running ahead as far
//        as the ring allows;
//      * warps 0-7 dequantize W: thread r takes row r's two Q4_0 blocks of
//        the stage, with the raw bytes of the next three stages already in
//        flight in registers, and store them as bf16 in the swizzled layout.
//      * warp 8 allocates BN tensor-memory columns; its lane 0 issues
//        tcgen05.mma (M = 128, N = BN, K = 16, bf16 -> fp32) four times per
//        stage and frees the stage with tcgen05.commit on the stage's
//        "empty" mbarrier; a last commit signals "done".
//      * warps 0-7 then read the accumulator (tcgen05.ld, 32 lanes x 32
//        columns at a time), add the bias and store C.
//   Every wait is bounded (1 s of %globaltimer). A wait that gives up sets a
//   CTA-wide abort flag and the workspace error word; the MMA issuer still
//   commits what it issued, and tensor memory is freed only after the last
//   commit has landed (or its own bounded wait gave up).
#include <cuda.h>  // CUtensorMap (the encoder is fetched at run time)

#include <algorithm>
#include <mutex>

#include "qg_internal.cuh"
#include "tcgen05_util.cuh"

namespace qg {
namespace gq4 {

using namespace tc;

constexpr int kBM = 128;
constexpr int kBK = 64;               // one 128-byte swizzle row of bf16
constexpr int kProducers = 256;       // warps 0-7: W
constexpr int kThreads = kProducers + 64;  // + warp 8 (MMA) + warp 9 (TMA for A)
constexpr int kPrefetch = 3;          // W stages in flight in registers

// BN output columns and MT 128-row sub-tiles of A per CTA: the MT sub-tiles
// share each dequantized W tile (MT MMAs per K step into MT * BN tensor-memory
// columns), so W is dequantized once per MT * 128 rows of A.
template <int BN, int MT>
struct Cfg {
  static constexpr int kStageA = MT * kBM * kBK * 2;  // 16 KB per sub-tile
  static constexpr int kStageB = BN * kBK * 2;        // 16 or 32 KB
  static constexpr int kStage = kStageA + kStageB;
  static constexpr int kStages = (192 * 1024) / kStage < 6 ? (192 * 1024) / kStage : 6;
  static constexpr int kSmem = 1024 + kStages * kStage + 1024;  // + align slack + barriers
  static constexpr int kTmemCols = MT * BN;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  return (uint32_t)f32_to_bf16_bits(lo) | ((uint32_t)f32_to_bf16_bits(hi) << 16);
}

__global__ void a_to_bf16_kernel(const float* __restrict__ A, uint32_t* __restrict__ Ab, size_t n4) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n4;
       i += (size_t)gridDim.x * blockDim.x) {
    const float4 v = reinterpret_cast<const float4*>(A)[i];
    uint2 o;
    o.x = pack_bf16x2(v.x, v.y);
    o.y = pack_bf16x2(v.z, v.w);
    reinterpret_cast<uint2*>(Ab)[i] = o;
  }
}



// dequantize two Q4_0 blocks (raw: 36 bytes as 9 words; fp16 d then 16 code
// bytes, twice) and store them as row r's 64 bf16 values of the stage. A
// nibble n becomes n - 8 exactly as float(0x4B000000 | n) - (2^23 + 8); the
// product with d is exact in fp32 and rounds once to bf16.
__device__ __forceinline__ float nib_m8(uint32_t w, int sh) {
  return __uint_as_float(0x4B000000u | ((w >> sh) & 0xFu)) - 8388616.0f;
}
__device__ __forceinline__ uint32_t bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}
__device__ __forceinline__ void store_w_row(uint8_t* sb, int r, const uint32_t (&raw)[9]) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    // block h: halfwords 9h .. 9h+8 of the 36 bytes
    auto hw = [&](int i) -> uint32_t {
      const int k = 9 * h + i;
      return (raw[k >> 1] >> (16 * (k & 1))) & 0xFFFFu;
    };
    const float d = __half2float(__ushort_as_half((unsigned short)hw(0)));
    float w[32];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const uint32_t b2 = hw(1 + q);  // code bytes 2q, 2q+1
      w[2 * q] = nib_m8(b2, 0) * d;
      w[2 * q + 1] = nib_m8(b2, 8) * d;
      w[2 * q + 16] = nib_m8(b2, 4) * d;
      w[2 * q + 17] = nib_m8(b2, 12) * d;
    }
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      const int c = h * 4 + cc;
      uint4 v;
      v.x = bf16x2(w[cc * 8 + 0], w[cc * 8 + 1]);
      v.y = bf16x2(w[cc * 8 + 2], w[cc * 8 + 3]);
      v.z = bf16x2(w[cc * 8 + 4], w[cc * 8 + 5]);
      v.w = bf16x2(w[cc * 8 + 6], w[cc * 8 + 7]);
      *reinterpret_cast<uint4*>(sb + r * 128 + ((c ^ (r & 7)) << 4)) = v;
    }
  }
}

// the 36 raw bytes of row `wrow`'s two blocks of stage kb: nine 32-bit loads
// when the bytes are 4-byte aligned (K % 64 == 0 makes every stage's offset a
// multiple of 36), else eighteen 16-bit loads
template <bool W32>
__device__ __forceinline__ void load_w_raw(const uint8_t* wrow, int kb, uint32_t (&raw)[9]) {
  if constexpr (W32) {
    const uint32_t* p = reinterpret_cast<const uint32_t*>(wrow + (size_t)kb * 36);
#pragma unroll
    for (int i = 0; i < 9; ++i) raw[i] = __ldg(p + i);
  } else {
    const uint16_t* p = reinterpret_cast<const uint16_t*>(wrow + (size_t)kb * 36);
#pragma unroll
    for (int i = 0; i < 9; ++i)
      raw[i] = (uint32_t)__ldg(p + 2 * i) | ((uint32_t)__ldg(p + 2 * i + 1) << 16);
  }
}

// What the epilogue does with an accumulator value v of C[m][n]:
// v + bias[n] (+ res[m][n]), then gelu_tanh when `gelu`, stored as fp32 or
// bf16 (round to nearest even). C may alias res (each element is read and
// written by the same thread).
struct Epi {
  const float* bias;  // [N] or null
  const float* res;   // fp32 [M][N] or null
  void* C;            // [M][N]
  int c_bf16;
  int gelu;
  // test of the timeout path (gemm_q4_0_tc_kernel only): no load is issued
  // and no producer arrives, so the MMA issuer's first wait runs out (after
  // 1 ms) with nothing in flight
  int stall;
};

// GELU, tanh form (fuel-transformers `gelu_tanh`), in fp32 with CUDA's tanhf
__device__ __forceinline__ float gelu_tanh_f(float x) {
  return 0.5f * x * (1.0f + tanhf(0.7978845608028654f * (x + 0.044715f * x * x * x)));
}

// The epilogue shared by both kernels: warps 0-7 wait (bounded) for the last
// commit, read the accumulator and store C through the Epi rules; then
// tensor memory is freed. `ok` is this thread's own status so far.
template <int BN, int MT>
__device__ __forceinline__ void epilogue(uint32_t tmem, uint64_t* done, volatile int* abort,
                                         const Epi& ep, int M, int N, int m0, int n0, int warp,
                                         int lane, bool ok, unsigned* err) {
  bool landed = true;
  if (warp < 8) {
    // wait for the last commit even after an abort: tensor memory may only
    // be read or freed once the MMAs writing it are done
    // one poller per warp so the (warp-collective) tensor-memory loads below
    // see one decision
    int st = 0;
    if (lane == 0) {
      bool l = mbar_try_wait(done, 0);
      if (!l) {
        const unsigned long long t0 = now_ns();
        while (!(l = mbar_try_wait(done, 0)))
          if (now_ns() - t0 > kWaitNs) break;
      }
      st = (l ? 1 : 0) | (*abort ? 2 : 0);
    }
    st = __shfl_sync(0xffffffffu, st, 0);
    landed = (st & 1) != 0;
    const bool aborted = (st & 2) != 0;
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (landed && !aborted) {
      // warp w reads tensor-memory lanes 32 (w % 4) .. +31 (its rows) and
      // half of the MT * BN accumulator columns
      const int q = warp & 3, half = warp >> 2;
      constexpr int kCols = MT * BN / 2;
#pragma unroll 1
      for (int c0 = half * kCols; c0 < (half + 1) * kCols; c0 += 32) {
        uint32_t v[32];
        const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)c0;
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
            "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
              "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
              "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]),
              "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
              "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]),
              "=r"(v[31])
            : "r"(ta));
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        const int mt = c0 / BN, n = c0 % BN;
        const int m = m0 + mt * kBM + 32 * q + lane;
        if (m < M) {
          const size_t ci = (size_t)m * N + n0 + n;
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            float o[4] = {__uint_as_float(v[j]), __uint_as_float(v[j + 1]),
                          __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3])};
            if (ep.bias) {
#pragma unroll
              for (int e = 0; e < 4; ++e) o[e] += ep.bias[n0 + n + j + e];
            }
            if (ep.res) {
              const float4 r = *reinterpret_cast<const float4*>(ep.res + ci + j);
              o[0] += r.x;
              o[1] += r.y;
              o[2] += r.z;
              o[3] += r.w;
            }
            if (ep.gelu) {
#pragma unroll
              for (int e = 0; e < 4; ++e) o[e] = gelu_tanh_f(o[e]);
            }
            if (ep.c_bf16)
              *reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(ep.C) + ci + j) =
                  make_uint2(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]));
            else
              *reinterpret_cast<float4*>(reinterpret_cast<float*>(ep.C) + ci + j) =
                  make_float4(o[0], o[1], o[2], o[3]);
          }
        }
      }
    }
    if (!landed || aborted) ok = false;
  }
  if (!ok && err) atomicOr(err, 1u);
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 8) {
    __syncwarp();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(MT * BN));
  }
}

template <int BN, int MT, bool W32>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_q4_0_tc_kernel(const __grid_constant__ CUtensorMap tmA, const uint8_t* __restrict__ blocks,
                        const Epi ep, int M, int N, int K, unsigned* __restrict__ err) {
  using G = Cfg<BN, MT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* stages = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + G::kStages * G::kStage);
  uint64_t* tfull = full + G::kStages;
  uint64_t* empty = tfull + G::kStages;
  uint64_t* done = empty + G::kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n0 = blockIdx.x * BN, m0 = blockIdx.y * (MT * kBM);
  const int nk = K / kBK;
  const size_t rowbytes = (size_t)(K / 32) * 18;

  if (tid == 0) {
    for (int s = 0; s < G::kStages; ++s) {
      mbar_init(&full[s], kProducers);
      mbar_init(&tfull[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 8) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(G::kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;

  bool ok = true;
  if (warp < 8) {
    // ------------------------------------------------------ W producers
    // (none of this runs when stalling: the timeout test)
    const bool has_row = tid < BN && !ep.stall;
    const int nkp = ep.stall ? 0 : nk;
    const uint8_t* wrow = blocks + (size_t)(n0 + (has_row ? tid : 0)) * rowbytes;
    uint32_t raw[kPrefetch][9];
#pragma unroll
    for (int u = 0; u < kPrefetch; ++u)
      if (has_row && u < nkp) load_w_raw<W32>(wrow, u, raw[u]);
    for (int kb0 = 0; kb0 < nkp && ok; kb0 += kPrefetch) {
#pragma unroll
      for (int u = 0; u < kPrefetch; ++u) {
        const int kb = kb0 + u;
        if (kb >= nkp) break;
        const int s = kb % G::kStages;
        if (kb >= G::kStages &&
            !wait_bar(&empty[s], (uint32_t)((kb / G::kStages) + 1) & 1u, abort)) {
          ok = false;
          break;
        }
        if (has_row) {
          store_w_row(stages + (size_t)s * G::kStage + G::kStageA, tid, raw[u]);
          if (kb + kPrefetch < nkp) load_w_raw<W32>(wrow, kb + kPrefetch, raw[u]);
        }
        // make the generic-proxy stores visible to the tensor core
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_arrive(&full[s]);
      }
    }
    if (!ok) *abort = 1;
  } else if (warp == 9) {
    // ------------------------------------------------- A by TMA (lane 0)
    if (lane == 0 && !ep.stall) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
      int issued = 0;
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % G::kStages;
        if (kb >= G::kStages &&
            !wait_bar(&empty[s], (uint32_t)((kb / G::kStages) + 1) & 1u, abort)) {
          ok = false;
          *abort = 1;
          break;
        }
        mbar_expect_tx(&tfull[s], (uint32_t)G::kStageA);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
          asm volatile(
              "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
              " [%0], [%1, {%2, %3}], [%4];" ::"r"(
                  smem_u32(stages + (size_t)s * G::kStage + mt * kBM * kBK * 2)),
              "l"(reinterpret_cast<uint64_t>(&tmA)), "r"(kb * kBK), "r"(m0 + mt * kBM),
              "r"(smem_u32(&tfull[s]))
              : "memory");
        ++issued;
      }
      // no copy may land after the CTA is gone: wait (bounded) for the last
      // fill of every stage used
      for (int j = issued - G::kStages > 0 ? issued - G::kStages : 0; j < issued; ++j) {
        const int s = j % G::kStages;
        const uint32_t par = (uint32_t)(j / G::kStages) & 1u;
        if (!mbar_try_wait(&tfull[s], par)) {
          const unsigned long long t0 = now_ns();
          while (!mbar_try_wait(&tfull[s], par))
            if (now_ns() - t0 > kWaitNs) break;
        }
      }
    }
  } else if (lane == 0) {
    // ------------------------------------------------------- MMA issuer
    const uint32_t idesc = instr_desc<BN>();
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % G::kStages;
      const uint32_t par = (uint32_t)(kb / G::kStages) & 1u;
      const unsigned long long lim = ep.stall ? 1000000ull : kWaitNs;
      if (!wait_bar_ns(&tfull[s], par, abort, lim) || !wait_bar_ns(&full[s], par, abort, lim)) {
        ok = false;
        *abort = 1;
        break;
      }
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t sa = smem_u32(stages + (size_t)s * G::kStage);
      const uint32_t sb = sa + G::kStageA;
#pragma unroll
      for (int k = 0; k < kBK / 16; ++k) {
        const uint64_t db = smem_desc(sb + k * 32);
        const uint32_t acc = (kb > 0 || k > 0) ? 1u : 0u;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          const uint64_t da = smem_desc(sa + mt * kBM * kBK * 2 + k * 32);
          asm volatile(
              "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
              " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
                  tmem + (uint32_t)(mt * BN)),
              "l"(da), "l"(db), "r"(idesc), "r"(acc)
              : "memory");
        }
      }
      asm volatile(
          "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
              smem_u32(&empty[s]))
          : "memory");
    }
    // completes once every MMA issued above has finished
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(done))
        : "memory");
  }

  epilogue<BN, MT>(tmem, done, abort, ep, M, N, m0, n0, warp, lane, ok, err);
}


// W's raw Q4_0 rows staged by TMA (K % 256 == 0, so every row's byte length
// is a multiple of 16): a box of kRawRow bytes a row covers four MMA stages
// (two Q4_0 blocks a stage).
constexpr int kRawStages = 4;                 // MMA stages per raw chunk
constexpr int kRawRow = kRawStages * 36;      // 144 bytes of a row per chunk

// ---------------------------------------------------------------------------
// Transposed form (K % 256 == 0). The tile is 128 rows of W by TN rows of A:
// D[n][m] = sum_k W[n][k] A[m][k], so W is the MMA's A operand and comes from
// tensor memory. The converter warps dequantize each stage's 128 x 64 block
// of W straight into a ring of tensor-memory stages with tcgen05.st (thread
// = W row = tensor-memory lane): no swizzled shared-memory stores, no proxy
// fence, and shared memory left for a deep ring of A's TN x 64 tiles, the B
// operand, staged by TMA with the 128-byte swizzle. Roles:
//   warps 0 .. kTConv-1  converters, then the epilogue. They form
//              kTGroups groups of 8 warps that take the stages in turn
//              (group g: stages k = g mod kTGroups), since one stage's
//              conversion is a chain of latencies (shared-memory loads, the
//              arithmetic, the tensor-memory store) rather than work; in a
//              group, warp w holds W rows 32 (w % 4) + lane of Q4_0 block
//              (w / 4) % 2. A converter issues stage k's store, converts its
//              next stage, and only then waits for the store and publishes
//              stage k;
//   warp kTConv  lane 0: TMA for A's stages;
//   warp kTConv+1  tensor-memory allocation; lane 0 issues four MMAs a
//              stage (M = 128, N = TN, K = 16, bf16 -> fp32) and commits;
//   warp kTConv+2  lane 0: TMA for W's raw rows (144 bytes a row = four
//              stages per chunk, a ring of kTRaw chunks), apart from A's
//              loads so that neither waits behind the other.
// A stage's A tile and W columns share one full/empty barrier pair, so the
// MMA thread has one wait and one commit a stage.
// ---------------------------------------------------------------------------
constexpr int kTConv = 16;                 // converter warps (16 or 24)
constexpr int kTGroups = kTConv / 8;       // converter groups, stages taken in turn
constexpr int kTEpi = 16;                  // the first kTEpi converter warps then run the epilogue
constexpr int kTThreads = 32 * (kTConv + 3);
constexpr bool kTPipe = false;             // publish a stage only after converting the next (measured slower)
constexpr int kTCols = 16;                 // tensor-memory columns a converter thread stores a stage
constexpr int kTRaw = 3;                   // raw W chunks in flight

template <int TN>
struct CfgT {
  static constexpr int kStageB = TN * kBK * 2;  // A's rows of a stage, bf16
  static constexpr int kRawSlot = kBM * kRawRow;  // 18 KB
  static constexpr int kRoom = 216 * 1024 - kTRaw * kRawSlot;
  static constexpr int kStages = kRoom / kStageB > 8 ? 8 : kRoom / kStageB;
  static constexpr int kSmem = 1024 + kStages * kStageB + kTRaw * kRawSlot + 512;
  static constexpr int kAccCols = TN;           // accumulator: columns [0, TN)
  // stage s of the ring: A's tile in shared memory and W's 32 tensor-memory
  // columns from kAccCols + 32 s, filled and freed together
  static_assert(TN + kStages * 32 <= 512, "tensor memory");
};

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// Q4_0 block H of a stage (halfwords 9H .. 9H + 8 of its 36 raw bytes: the
// fp16 d, then 16 code bytes) as bf16 pairs in k order, pair j = values
// 2j, 2j + 1: values 0-15 are the low nibbles of code bytes 0-15 (pairs
// 0-7), values 16-31 the high ones (pairs 8-15). Each value (n - 8) d is
// exact in fp32 and rounds once to bf16, as in store_w_row.
template <int H>
__device__ __forceinline__ void w_block_pairs(const uint32_t (&raw)[9], uint32_t (&v)[16]) {
  auto hw = [&](int i) -> uint32_t {
    const int k = 9 * H + i;
    return (raw[k >> 1] >> (16 * (k & 1))) & 0xFFFFu;
  };
  const float d = __half2float(__ushort_as_half((unsigned short)hw(0)));
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const uint32_t b2 = hw(1 + q);  // code bytes 2q, 2q + 1
    v[q] = bf16x2(nib_m8(b2, 0) * d, nib_m8(b2, 8) * d);
    v[q + 8] = bf16x2(nib_m8(b2, 4) * d, nib_m8(b2, 12) * d);
  }
}
// a converter's 16 pairs of a stage: Q4_0 block p (columns 16 p .. 16 p + 15)
__device__ __forceinline__ void w_stage_pairs(const uint32_t (&raw)[9], int p, uint32_t (&v)[16]) {
  if (p == 0) w_block_pairs<0>(raw, v);
  else w_block_pairs<1>(raw, v);
}
__device__ __forceinline__ void tmem_st_pairs(uint32_t ta, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16};" ::"r"(ta),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15])
      : "memory");
}

// The epilogue of the transposed tile: warp w reads tensor-memory lanes
// 32 (w % 4) .. +31 (W rows n, columns of C) and half of the TN columns
// (A rows m); each value goes through the Epi rules to C[m][n] (a warp's
// stores for one m are 32 consecutive n).
template <int TN>
__device__ __forceinline__ void epilogue_t(uint32_t tmem, uint64_t* done, volatile int* abort,
                                           const Epi& ep, int M, int N, int m0, int n0, int warp,
                                           int lane, bool ok, unsigned* err) {
  bool landed = true;
  if (warp < kTEpi) {
    int st = 0;
    if (lane == 0) {
      bool l = mbar_try_wait(done, 0);
      if (!l) {
        const unsigned long long t0 = now_ns();
        while (!(l = mbar_try_wait(done, 0)))
          if (now_ns() - t0 > kWaitNs) break;
      }
      st = (l ? 1 : 0) | (*abort ? 2 : 0);
    }
    st = __shfl_sync(0xffffffffu, st, 0);
    landed = (st & 1) != 0;
    const bool aborted = (st & 2) != 0;
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (landed && !aborted) {
      const int q = warp & 3, part = warp >> 2;
      const int n = n0 + 32 * q + lane;
      const float bias = ep.bias ? ep.bias[n] : 0.f;
      // this warp's kCols columns in rounds of 64: both 32-column loads of a
      // round are in flight before the one wait
      constexpr int kCols = TN / (kTEpi / 4);
      constexpr int kRound = kCols < 64 && kTConv <= 16 ? kCols : (kTConv <= 16 ? 64 : 32);
#pragma unroll 1
      for (int c0 = part * kCols; c0 < (part + 1) * kCols; c0 += kRound) {
        if (m0 + c0 >= M) break;
        uint32_t v[kRound];
#pragma unroll
        for (int hb = 0; hb < kRound / 32; ++hb) {
          const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(c0 + 32 * hb);
          uint32_t* w = v + 32 * hb;
          asm volatile(
              "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
              "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
              : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]),
                "=r"(w[6]), "=r"(w[7]), "=r"(w[8]), "=r"(w[9]), "=r"(w[10]), "=r"(w[11]),
                "=r"(w[12]), "=r"(w[13]), "=r"(w[14]), "=r"(w[15]), "=r"(w[16]), "=r"(w[17]),
                "=r"(w[18]), "=r"(w[19]), "=r"(w[20]), "=r"(w[21]), "=r"(w[22]), "=r"(w[23]),
                "=r"(w[24]), "=r"(w[25]), "=r"(w[26]), "=r"(w[27]), "=r"(w[28]), "=r"(w[29]),
                "=r"(w[30]), "=r"(w[31])
              : "r"(ta));
        }
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
        for (int j = 0; j < kRound; ++j) {
          const int m = m0 + c0 + j;
          if (m < M) {
            const size_t ci = (size_t)m * N + n;
            float o = __uint_as_float(v[j]);
            if (ep.bias) o += bias;
            if (ep.res) o += ep.res[ci];
            if (ep.gelu) o = gelu_tanh_f(o);
            if (ep.c_bf16)
              reinterpret_cast<uint16_t*>(ep.C)[ci] = f32_to_bf16_bits(o);
            else
              reinterpret_cast<float*>(ep.C)[ci] = o;
          }
        }
      }
    }
    if (!landed || aborted) ok = false;
  }
  if (!ok && err) atomicOr(err, 1u);
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == kTConv + 1) {
    __syncwarp();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

// no copy may land after the CTA is gone: wait (bounded) for the last fill of
// every slot of a ring (count fills issued over nslots slots)
__device__ __forceinline__ void tma_drain(uint64_t* bars, int nslots, int count) {
  for (int j = count - nslots > 0 ? count - nslots : 0; j < count; ++j) {
    const int s = j % nslots;
    const uint32_t par = (uint32_t)(j / nslots) & 1u;
    if (!mbar_try_wait(&bars[s], par)) {
      const unsigned long long t0 = now_ns();
      while (!mbar_try_wait(&bars[s], par))
        if (now_ns() - t0 > kWaitNs) break;
    }
  }
}

template <int TN>
__global__ void __launch_bounds__(kTThreads, 1)
    gemm_q4_0_t_kernel(const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmW, const Epi ep, int M, int N, int K,
                       unsigned* __restrict__ err) {
  using G = CfgT<TN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* bst = smem;                                 // A's stages (the MMA's B operand)
  uint8_t* raws = smem + G::kStages * G::kStageB;      // W's raw chunks
  // full[s]: A's tile landed (TMA bytes) and W's stage converted; empty[s]:
  // the MMAs reading both are done (one commit)
  uint64_t* full = reinterpret_cast<uint64_t*>(raws + kTRaw * G::kRawSlot);
  uint64_t* empty = full + G::kStages;
  uint64_t* rfull = empty + G::kStages;
  uint64_t* rempty = rfull + kTRaw;
  uint64_t* done = rempty + kTRaw;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n0 = blockIdx.x * kBM, m0 = blockIdx.y * TN;
  const int nk = K / kBK, nchunk = nk / kRawStages;  // K % 256 == 0

  if (tid == 0) {
    for (int s = 0; s < G::kStages; ++s) {
      mbar_init(&full[s], 32 * 8 + 1);  // the converting group and the TMA's arrival
      mbar_init(&empty[s], 1);
    }
    for (int r = 0; r < kTRaw; ++r) {
      mbar_init(&rfull[r], 1);
      mbar_init(&rempty[r], 32 * kTConv);  // every group reads every chunk
    }
    mbar_init(done, 1);
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kTConv + 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;

  bool ok = true;
  if (warp < kTConv) {
    // ------------------------------------------------------ converters
    const int q = warp & 3, p = (warp >> 2) & 1, grp = warp >> 3, r = 32 * q + lane;
    // stage k is published (its store waited for, the ring slots released)
    // once the group's next stage has been converted
    auto publish = [&](int k) {
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      // the raw chunk is consumed once the stores have used its last
      // stage's values
      if (k % kRawStages + kTGroups >= kRawStages)  // the group's last stage of the chunk
        mbar_arrive(&rempty[(k / kRawStages) % kTRaw]);  // (every group has one: 4 >= groups)
      mbar_arrive(&full[k % G::kStages]);
    };
    int pend = -1;  // stage whose store is issued but not yet published
    for (int kb = grp; kb < nk; kb += kTGroups) {
      const int c = kb / kRawStages, sub = kb % kRawStages, slot = c % kTRaw, a = kb % G::kStages;
      // (sub < kTGroups: the group's first stage of the chunk)
      if ((sub < kTGroups && !wait_bar(&rfull[slot], (uint32_t)(c / kTRaw) & 1u, abort)) ||
          (kb >= G::kStages &&
           !wait_bar(&empty[a], (uint32_t)((kb / G::kStages) + 1) & 1u, abort))) {
        ok = false;
        break;
      }
      const uint32_t* rw =
          reinterpret_cast<const uint32_t*>(raws + slot * G::kRawSlot + r * kRawRow + sub * 36);
      uint32_t raw[9];
#pragma unroll
      for (int i = 0; i < 9; ++i) raw[i] = rw[i];
      uint32_t v[kTCols];
      w_stage_pairs(raw, p, v);
      if (pend >= 0) publish(pend);
      tmem_st_pairs(tmem + ((uint32_t)(32 * q) << 16) +
                        (uint32_t)(G::kAccCols + a * 32 + p * kTCols),
                    v);
      pend = kb;
      // the first stage goes out at once: the MMA has nothing else to do yet
      if (!kTPipe || kb < kTGroups) {
        publish(kb);
        pend = -1;
      }
    }
    if (ok && pend >= 0) publish(pend);
    if (!ok) *abort = 1;
  } else if (warp == kTConv) {
    // ----------------------- A's stages by TMA (lane 0), as far ahead as the ring allows
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
      int issued = 0;
      for (int kb = 0; kb < nk && ok; ++kb) {
        const int s = kb % G::kStages;
        if (kb >= G::kStages &&
            !wait_bar(&empty[s], (uint32_t)((kb / G::kStages) + 1) & 1u, abort)) {
          ok = false;
          break;
        }
        mbar_expect_tx(&full[s], (uint32_t)G::kStageB);  // (the TMA's arrival)
        tma_load_2d(smem_u32(bst + (size_t)s * G::kStageB), &tmA, kb * kBK, m0, &full[s]);
        ++issued;
      }
      if (!ok) *abort = 1;
      tma_drain(full, G::kStages, issued);
    }
  } else if (warp == kTConv + 2) {
    // ------------------------------------ W's raw chunks by TMA (lane 0)
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmW)) : "memory");
      int rissued = 0;
      for (int c = 0; c < nchunk && ok; ++c) {
        const int slot = c % kTRaw;
        if (c >= kTRaw && !wait_bar(&rempty[slot], (uint32_t)((c / kTRaw) + 1) & 1u, abort)) {
          ok = false;
          break;
        }
        mbar_expect_tx(&rfull[slot], (uint32_t)G::kRawSlot);
        tma_load_2d(smem_u32(raws + slot * G::kRawSlot), &tmW, c * kRawRow, n0, &rfull[slot]);
        ++rissued;
      }
      if (!ok) *abort = 1;
      tma_drain(rfull, kTRaw, rissued);
    }
  } else if (warp == kTConv + 1 && lane == 0) {
    // ------------------------------------------------------- MMA issuer
    const uint32_t idesc = instr_desc<TN>();
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % G::kStages;
      if (!wait_bar(&full[s], (uint32_t)(kb / G::kStages) & 1u, abort)) {
        ok = false;
        *abort = 1;
        break;
      }
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      // K step k starts 32 bytes further: 2 in the descriptor's address field
      const uint64_t db0 = smem_desc(smem_u32(bst + (size_t)s * G::kStageB));
      const uint32_t ta = tmem + (uint32_t)(G::kAccCols + s * 32);
#pragma unroll
      for (int k = 0; k < kBK / 16; ++k) {
        const uint64_t db = db0 + (uint64_t)(2 * k);
        const uint32_t acc = (kb > 0 || k > 0) ? 1u : 0u;
        asm volatile(
            "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
            " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(tmem),
            "r"(ta + (uint32_t)(k * 8)), "l"(db), "r"(idesc), "r"(acc)
            : "memory");
      }
      asm volatile(
          "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
              smem_u32(&empty[s]))
          : "memory");
    }
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(done))
        : "memory");
  }
  epilogue_t<TN>(tmem, done, abort, ep, M, N, m0, n0, warp, lane, ok, err);
}
}  // namespace gq4

static size_t a_bytes(int M, int K) { return (((size_t)M * K * 2) + 255) & ~(size_t)255; }

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// the driver's tensor-map encoder, fetched once through the runtime
static EncodeTiledFn encode_tiled() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// A bf16 [rows][cols] row-major tensor (row stride cols * 2 bytes) in boxes
// of 64 columns x box_rows rows, 128-byte swizzle; rows past the end read as
// zero.
bool make_bf16_map(CUtensorMap* map, const void* base, int rows, int cols, int box_rows) {
  EncodeTiledFn enc = encode_tiled();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A byte [rows][cols] row-major tensor (row stride cols bytes, a multiple
// of 16) in boxes of box_cols x box_rows, with no swizzle or the 128-byte
// one (box_cols = 128: 16-byte chunk c of a box row r lands at chunk
// c ^ (r % 8)); bytes past the end read as zero.
bool make_u8_map(CUtensorMap* map, const void* base, int rows, int cols, int box_cols,
                 int box_rows, bool swizzle128) {
  EncodeTiledFn enc = encode_tiled();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols};
  const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static bool make_a_map(CUtensorMap* map, const uint16_t* Ab, int M, int K) {
  return make_bf16_map(map, Ab, M, K, gq4::kBM);
}

template <int BN, int MT, bool W32>
static cudaError_t gq4_launch(const CUtensorMap& tmA, const uint8_t* blocks, const gq4::Epi& ep,
                              int M, int N, int K, unsigned* err, cudaStream_t st) {
  using G = gq4::Cfg<BN, MT>;
  ensure_smem((const void*)gq4::gemm_q4_0_tc_kernel<BN, MT, W32>, G::kSmem);
  dim3 grid(N / BN, (M + MT * gq4::kBM - 1) / (MT * gq4::kBM));
  return launch_pdl(gq4::gemm_q4_0_tc_kernel<BN, MT, W32>, grid, dim3(gq4::kThreads),
                    (size_t)G::kSmem, st, false, tmA, blocks, ep, M, N, K, err);
}

// tile choice: 256 columns when N allows; two A sub-tiles per CTA (W
// dequantized once per 256 rows of A) while that still gives half the SMs a
// tile
template <int BN, bool W32>
static cudaError_t gq4_launch_mt(const CUtensorMap& tmA, const uint8_t* blocks, const gq4::Epi& ep,
                                 int M, int N, int K, unsigned* err, cudaStream_t st) {
  const long long tiles2 = (long long)(N / BN) * ((M + 255) / 256);
  if (2 * tiles2 >= num_sms())
    return gq4_launch<BN, 2, W32>(tmA, blocks, ep, M, N, K, err, st);
  return gq4_launch<BN, 1, W32>(tmA, blocks, ep, M, N, K, err, st);
}

// W's raw Q4_0 rows ([N][K/32 * 18] bytes; K % 256 == 0 makes the row
// stride a multiple of 16) in boxes of 144 bytes (four MMA stages) x BN rows;
// bytes past a row's end read as zero.
static bool make_w_raw_map(CUtensorMap* map, const uint8_t* blocks, int N, int K, int BN) {
  EncodeTiledFn enc = encode_tiled();
  if (!enc) return false;
  const cuuint64_t rowbytes = (cuuint64_t)(K / 32) * 18;
  const cuuint64_t dims[2] = {rowbytes, (cuuint64_t)N};
  const cuuint64_t strides[1] = {rowbytes};
  const cuuint32_t box[2] = {(cuuint32_t)gq4::kRawRow, (cuuint32_t)BN};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(blocks), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int TN>
static cudaError_t gq4_launch_t(const CUtensorMap& tmA, const CUtensorMap& tmW, const gq4::Epi& ep,
                                int M, int N, int K, unsigned* err, cudaStream_t st) {
  using G = gq4::CfgT<TN>;
  ensure_smem((const void*)gq4::gemm_q4_0_t_kernel<TN>, G::kSmem);
  dim3 grid(N / gq4::kBM, (M + TN - 1) / TN);
  return launch_pdl(gq4::gemm_q4_0_t_kernel<TN>, grid, dim3(gq4::kTThreads), (size_t)G::kSmem, st,
                    false, tmA, tmW, ep, M, N, K, err);
}

// The GEMM on a bf16 A already in device memory (`Ab`, [M][K]); `err` is the
// workspace error word.
static qg_status gq4_run(const uint8_t* blocks, const uint16_t* Ab, const gq4::Epi& ep, int M,
                         int N, int K, unsigned* err, cudaStream_t s, const char* what) {
  if (K % 256 == 0 && aligned(blocks, 16)) {
    // the transposed form: W's raw rows and A's tiles staged by TMA, W
    // dequantized into tensor memory; 256 rows of A a tile while that still
    // fills the SMs, else 128
    const int TN = (long long)(N / gq4::kBM) * ((M + 255) / 256) >= num_sms() ? 256 : 128;
    CUtensorMap tmA, tmW;
    if (!make_bf16_map(&tmA, Ab, M, K, TN) || !make_w_raw_map(&tmW, blocks, N, K, gq4::kBM)) {
      set_error("%s: could not encode a TMA descriptor", what);
      return QG_ERR_CUDA;
    }
    if (TN == 256) gq4_launch_t<256>(tmA, tmW, ep, M, N, K, err, s);
    else gq4_launch_t<128>(tmA, tmW, ep, M, N, K, err, s);
    return check_launch(what);
  }
  CUtensorMap tmA;
  if (!make_a_map(&tmA, Ab, M, K)) {
    set_error("%s: could not encode the TMA descriptor of A", what);
    return QG_ERR_CUDA;
  }
  const bool w32 = aligned(blocks, 4);
  if (N % 256 == 0) {
    if (w32) gq4_launch_mt<256, true>(tmA, blocks, ep, M, N, K, err, s);
    else gq4_launch_mt<256, false>(tmA, blocks, ep, M, N, K, err, s);
  } else {
    if (w32) gq4_launch_mt<128, true>(tmA, blocks, ep, M, N, K, err, s);
    else gq4_launch_mt<128, false>(tmA, blocks, ep, M, N, K, err, s);
  }
  return check_launch(what);
}

}  // namespace qg

using namespace qg;

extern "C" size_t qg_gemm_q4_0_workspace_size(int M, int N, int K) {
  (void)N;
  if (M <= 0 || K <= 0) return 256;
  return a_bytes(M, K) + 256;
}

static qg_status gemm_q4_0_checked(const uint8_t* blocks, const void* A, qg_dtype a_dtype,
                                   const float* bias, const float* residual, void* C,
                                   qg_dtype c_dtype, int gelu, int M, int N, int K, void* ws,
                                   size_t ws_bytes, void* stream, const char* what) {
  clear_error();
  QG_REQUIRE(M >= 0 && N >= 0 && K >= 0, QG_ERR_UNSUPPORTED_SHAPE,
             "%s: M=%d N=%d K=%d must be >= 0", what, M, N, K);
  QG_REQUIRE(K % 64 == 0 && K > 0, QG_ERR_UNSUPPORTED_SHAPE,
             "%s: K=%d must be a positive multiple of 64", what, K);
  QG_REQUIRE(N % 128 == 0 && N > 0, QG_ERR_UNSUPPORTED_SHAPE,
             "%s: N=%d must be a positive multiple of 128", what, N);
  QG_REQUIRE((long long)M * K < (1LL << 40) && (long long)M * N < (1LL << 40),
             QG_ERR_UNSUPPORTED_SHAPE, "%s: M=%d too large", what, M);
  QG_REQUIRE(M < (1 << 24) / 128 * 128, QG_ERR_UNSUPPORTED_SHAPE, "%s: M=%d too large", what, M);
  QG_REQUIRE(a_dtype == QG_F32 || a_dtype == QG_BF16, QG_ERR_INVALID_ARGUMENT,
             "%s: a_dtype=%d", what, (int)a_dtype);
  QG_REQUIRE(c_dtype == QG_F32 || c_dtype == QG_BF16, QG_ERR_INVALID_ARGUMENT,
             "%s: c_dtype=%d", what, (int)c_dtype);
  QG_REQUIRE(!residual || c_dtype == QG_F32, QG_ERR_INVALID_ARGUMENT,
             "%s: a residual needs an fp32 C", what);
  if (M == 0) return QG_OK;
  QG_REQUIRE(blocks && A && C, QG_ERR_INVALID_ARGUMENT, "%s: null blocks, A or C", what);
  QG_REQUIRE(aligned(A, 16) && aligned(C, 16) && aligned(residual, 16), QG_ERR_MISALIGNED,
             "%s: A, C and residual must be 16-byte aligned", what);
  QG_REQUIRE(aligned(blocks, 2), QG_ERR_MISALIGNED, "%s: blocks must be 2-byte aligned", what);
  QG_REQUIRE(!bias || aligned(bias, 4), QG_ERR_MISALIGNED, "%s: bias misaligned", what);
  const size_t need = a_dtype == QG_F32 ? qg_gemm_q4_0_workspace_size(M, N, K) : 256;
  QG_REQUIRE(ws && ws_bytes >= need, QG_ERR_WORKSPACE_TOO_SMALL,
             "%s: workspace of %zu bytes given, %zu needed", what, ws_bytes, need);
  QG_REQUIRE(aligned(ws, 256), QG_ERR_MISALIGNED, "%s: ws not 256-byte aligned", what);
  cudaStream_t s = (cudaStream_t)stream;
  const uint16_t* Ab = reinterpret_cast<const uint16_t*>(A);
  unsigned* err = reinterpret_cast<unsigned*>(ws);
  if (a_dtype == QG_F32) {
    uint16_t* Aw = reinterpret_cast<uint16_t*>(ws);
    err = reinterpret_cast<unsigned*>(reinterpret_cast<uint8_t*>(ws) + a_bytes(M, K));
    const size_t n4 = (size_t)M * K / 4;
    const int grid = (int)std::min<size_t>((n4 + 255) / 256, (size_t)num_sms() * 8);
    launch_pdl(gq4::a_to_bf16_kernel, dim3(grid), dim3(256), 0, s, false,
               reinterpret_cast<const float*>(A), reinterpret_cast<uint32_t*>(Aw), n4);
    Ab = Aw;
  }
  cudaMemsetAsync(err, 0, sizeof(unsigned), s);
  gq4::Epi ep = {bias, residual, C, c_dtype == QG_BF16 ? 1 : 0, gelu ? 1 : 0, 0};
  return gq4_run(blocks, Ab, ep, M, N, K, err, s, what);
}

extern "C" qg_status qg_gemm_q4_0(const uint8_t* blocks, const float* A, const float* bias,
                                  float* C, int M, int N, int K, void* ws, size_t ws_bytes,
                                  void* stream) {
  return gemm_q4_0_checked(blocks, A, QG_F32, bias, nullptr, C, QG_F32, 0, M, N, K, ws, ws_bytes,
                           stream, "qg_gemm_q4_0");
}

extern "C" qg_status qg_gemm_q4_0_ex(const uint8_t* blocks, const void* A, qg_dtype a_dtype,
                                     const float* bias, const float* residual, void* C,
                                     qg_dtype c_dtype, int gelu, int M, int N, int K, void* ws,
                                     size_t ws_bytes, void* stream) {
  return gemm_q4_0_checked(blocks, A, a_dtype, bias, residual, C, c_dtype, gelu, M, N, K, ws,
                           ws_bytes, stream, "qg_gemm_q4_0_ex");
}

extern "C" qg_status qg_gemm_q4_0_error(int M, int K, const void* ws, unsigned* code,
                                        void* stream) {
  clear_error();
  QG_REQUIRE(ws && code && M >= 0 && K >= 0, QG_ERR_INVALID_ARGUMENT,
             "qg_gemm_q4_0_error: null ws or code, or negative shape");
  cudaStream_t s = (cudaStream_t)stream;
  // after an fp32-A call the word follows A's bf16 copy; after a bf16-A
  // call (M = K = 0 here) it heads the workspace
  const size_t off = (M > 0 && K > 0) ? a_bytes(M, K) : 0;
  cudaError_t e = cudaMemcpyAsync(code, reinterpret_cast<const uint8_t*>(ws) + off,
                                  sizeof(unsigned), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    set_error("qg_gemm_q4_0_error: %s", cudaGetErrorString(e));
    return QG_ERR_CUDA;
  }
  if (*code != 0) {
    set_error("qg_gemm_q4_0: a device-side wait gave up (code 0x%x)", *code);
    return QG_ERR_TIMEOUT;
  }
  return QG_OK;
}

extern "C" qg_status qg_gemm_q4_0_stall_test(const uint8_t* blocks, const uint16_t* A, float* C,
                                             int M, int N, int K, void* ws, size_t ws_bytes,
                                             void* stream) {
  clear_error();
  QG_REQUIRE(M > 0 && N > 0 && N % 128 == 0 && K > 0 && K % 64 == 0, QG_ERR_UNSUPPORTED_SHAPE,
             "qg_gemm_q4_0_stall_test: M=%d N=%d K=%d", M, N, K);
  QG_REQUIRE(blocks && A && C && aligned(A, 16) && aligned(C, 16) && aligned(blocks, 4),
             QG_ERR_INVALID_ARGUMENT, "qg_gemm_q4_0_stall_test: bad pointer");
  QG_REQUIRE(ws && ws_bytes >= 256 && aligned(ws, 256), QG_ERR_WORKSPACE_TOO_SMALL,
             "qg_gemm_q4_0_stall_test: ws must be 256 bytes, 256-byte aligned");
  cudaStream_t s = (cudaStream_t)stream;
  unsigned* err = reinterpret_cast<unsigned*>(ws);
  cudaMemsetAsync(err, 0, sizeof(unsigned), s);
  CUtensorMap tmA;
  if (!make_a_map(&tmA, A, M, K)) {
    set_error("qg_gemm_q4_0_stall_test: could not encode the TMA descriptor of A");
    return QG_ERR_CUDA;
  }
  gq4::Epi ep = {nullptr, nullptr, C, 0, 0, 1};
  if (N % 256 == 0) gq4_launch<256, 1, true>(tmA, blocks, ep, M, N, K, err, s);
  else gq4_launch<128, 1, true>(tmA, blocks, ep, M, N, K, err, s);
  return check_launch("qg_gemm_q4_0_stall_test");
}
