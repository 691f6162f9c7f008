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
//   2. gemm_q4_0_tc_kernel, one CTA per 128 x BN output tile, over a ring of
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

namespace qg {
namespace gq4 {

constexpr int kBM = 128;
constexpr int kBK = 64;               // one 128-byte swizzle row of bf16
constexpr int kProducers = 256;       // warps 0-7: W
constexpr int kThreads = kProducers + 64;  // + warp 8 (MMA) + warp 9 (TMA for A)
constexpr int kPrefetch = 3;          // W stages in flight in registers
constexpr unsigned long long kWaitNs = 1000000000ull;

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

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
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
__device__ __forceinline__ unsigned long long now_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// bounded wait; gives up early once another role has aborted
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = now_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort) return false;
    if (now_ns() - t0 > kWaitNs) return false;
  }
  return true;
}

// K-major, 128-byte swizzle shared-memory matrix descriptor: 8-row groups
// 1024 bytes apart (SBO), leading offset 16 bytes, descriptor version 1.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;             // LBO = 16 B (encoded >> 4)
  d |= (uint64_t)(1024u >> 4) << 32;   // SBO = 1024 B
  d |= (uint64_t)1u << 46;             // version
  d |= (uint64_t)2u << 61;             // SWIZZLE_128B
  return d;
}

// instruction descriptor: bf16 x bf16 -> fp32, both K-major, M = 128
template <int BN>
__host__ __device__ constexpr uint32_t instr_desc() {
  return (1u << 4)                 // D fp32
         | (1u << 7)               // A bf16
         | (1u << 10)              // B bf16
         | ((uint32_t)(BN >> 3) << 17)
         | ((uint32_t)(kBM >> 4) << 24);
}

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

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
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

template <int BN, int MT, bool W32>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_q4_0_tc_kernel(const __grid_constant__ CUtensorMap tmA, const uint8_t* __restrict__ blocks,
                        const float* __restrict__ bias, float* __restrict__ C, int M, int N, int K,
                        unsigned* __restrict__ err) {
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
    const bool has_row = tid < BN;
    const uint8_t* wrow = blocks + (size_t)(n0 + (has_row ? tid : 0)) * rowbytes;
    uint32_t raw[kPrefetch][9];
#pragma unroll
    for (int u = 0; u < kPrefetch; ++u)
      if (has_row && u < nk) load_w_raw<W32>(wrow, u, raw[u]);
    for (int kb0 = 0; kb0 < nk && ok; kb0 += kPrefetch) {
#pragma unroll
      for (int u = 0; u < kPrefetch; ++u) {
        const int kb = kb0 + u;
        if (kb >= nk) break;
        const int s = kb % G::kStages;
        if (kb >= G::kStages &&
            !wait_bar(&empty[s], (uint32_t)((kb / G::kStages) + 1) & 1u, abort)) {
          ok = false;
          break;
        }
        if (has_row) {
          store_w_row(stages + (size_t)s * G::kStage + G::kStageA, tid, raw[u]);
          if (kb + kPrefetch < nk) load_w_raw<W32>(wrow, kb + kPrefetch, raw[u]);
        }
        // make the generic-proxy stores visible to the tensor core
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_arrive(&full[s]);
      }
    }
    if (!ok) *abort = 1;
  } else if (warp == 9) {
    // ------------------------------------------------- A by TMA (lane 0)
    if (lane == 0) {
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
      if (!wait_bar(&tfull[s], par, abort) || !wait_bar(&full[s], par, abort)) {
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

  // ---------------------------------------------------------- epilogue
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
          float* crow = C + (size_t)m * N + n0 + n;
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            float4 o = make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]),
                                   __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
            if (bias) {
              o.x += bias[n0 + n + j];
              o.y += bias[n0 + n + j + 1];
              o.z += bias[n0 + n + j + 2];
              o.w += bias[n0 + n + j + 3];
            }
            *reinterpret_cast<float4*>(crow + j) = o;
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
                 "r"(G::kTmemCols));
  }
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

// A (bf16 [M][K], row stride K*2 bytes) in boxes of 64 columns x 128 rows,
// 128-byte swizzle; rows past M read as zero
static bool make_a_map(CUtensorMap* map, const uint16_t* Ab, int M, int K) {
  EncodeTiledFn enc = encode_tiled();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
  const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  const cuuint32_t box[2] = {(cuuint32_t)gq4::kBK, (cuuint32_t)gq4::kBM};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(Ab), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN, int MT, bool W32>
static cudaError_t gq4_launch(const CUtensorMap& tmA, const uint8_t* blocks, const float* bias,
                              float* C, int M, int N, int K, unsigned* err, cudaStream_t st) {
  using G = gq4::Cfg<BN, MT>;
  ensure_smem((const void*)gq4::gemm_q4_0_tc_kernel<BN, MT, W32>, G::kSmem);
  dim3 grid(N / BN, (M + MT * gq4::kBM - 1) / (MT * gq4::kBM));
  return launch_pdl(gq4::gemm_q4_0_tc_kernel<BN, MT, W32>, grid, dim3(gq4::kThreads),
                    (size_t)G::kSmem, st, false, tmA, blocks, bias, C, M, N, K, err);
}

// tile choice: 256 columns when N allows; two A sub-tiles per CTA (W
// dequantized once per 256 rows of A) while that still gives half the SMs a
// tile
template <int BN, bool W32>
static cudaError_t gq4_launch_mt(const CUtensorMap& tmA, const uint8_t* blocks, const float* bias,
                                 float* C, int M, int N, int K, unsigned* err, cudaStream_t st) {
  const long long tiles2 = (long long)(N / BN) * ((M + 255) / 256);
  if (2 * tiles2 >= num_sms())
    return gq4_launch<BN, 2, W32>(tmA, blocks, bias, C, M, N, K, err, st);
  return gq4_launch<BN, 1, W32>(tmA, blocks, bias, C, M, N, K, err, st);
}

}  // namespace qg

using namespace qg;

extern "C" size_t qg_gemm_q4_0_workspace_size(int M, int N, int K) {
  (void)N;
  if (M <= 0 || K <= 0) return 256;
  return a_bytes(M, K) + 256;
}

extern "C" qg_status qg_gemm_q4_0(const uint8_t* blocks, const float* A, const float* bias,
                                  float* C, int M, int N, int K, void* ws, size_t ws_bytes,
                                  void* stream) {
  clear_error();
  QG_REQUIRE(M >= 0 && N >= 0 && K >= 0, QG_ERR_UNSUPPORTED_SHAPE,
             "qg_gemm_q4_0: M=%d N=%d K=%d must be >= 0", M, N, K);
  QG_REQUIRE(K % 64 == 0 && K > 0, QG_ERR_UNSUPPORTED_SHAPE,
             "qg_gemm_q4_0: K=%d must be a positive multiple of 64", K);
  QG_REQUIRE(N % 128 == 0 && N > 0, QG_ERR_UNSUPPORTED_SHAPE,
             "qg_gemm_q4_0: N=%d must be a positive multiple of 128", N);
  QG_REQUIRE((long long)M * K < (1LL << 40) && (long long)M * N < (1LL << 40),
             QG_ERR_UNSUPPORTED_SHAPE, "qg_gemm_q4_0: M=%d too large", M);
  QG_REQUIRE(M < (1 << 24) / 128 * 128, QG_ERR_UNSUPPORTED_SHAPE, "qg_gemm_q4_0: M=%d too large",
             M);
  if (M == 0) return QG_OK;
  QG_REQUIRE(blocks && A && C, QG_ERR_INVALID_ARGUMENT, "qg_gemm_q4_0: null blocks, A or C");
  QG_REQUIRE(aligned(A, 16) && aligned(C, 16), QG_ERR_MISALIGNED,
             "qg_gemm_q4_0: A and C must be 16-byte aligned");
  QG_REQUIRE(aligned(blocks, 2), QG_ERR_MISALIGNED, "qg_gemm_q4_0: blocks must be 2-byte aligned");
  QG_REQUIRE(!bias || aligned(bias, 4), QG_ERR_MISALIGNED, "qg_gemm_q4_0: bias misaligned");
  const size_t need = qg_gemm_q4_0_workspace_size(M, N, K);
  QG_REQUIRE(ws && ws_bytes >= need, QG_ERR_WORKSPACE_TOO_SMALL,
             "qg_gemm_q4_0: workspace of %zu bytes given, %zu needed", ws_bytes, need);
  QG_REQUIRE(aligned(ws, 256), QG_ERR_MISALIGNED, "qg_gemm_q4_0: ws not 256-byte aligned");
  cudaStream_t s = (cudaStream_t)stream;
  uint16_t* Ab = reinterpret_cast<uint16_t*>(ws);
  unsigned* err = reinterpret_cast<unsigned*>(reinterpret_cast<uint8_t*>(ws) + a_bytes(M, K));
  cudaMemsetAsync(err, 0, sizeof(unsigned), s);
  const size_t n4 = (size_t)M * K / 4;
  const int grid = (int)std::min<size_t>((n4 + 255) / 256, (size_t)num_sms() * 8);
  launch_pdl(gq4::a_to_bf16_kernel, dim3(grid), dim3(256), 0, s, false, A,
             reinterpret_cast<uint32_t*>(Ab), n4);
  CUtensorMap tmA;
  if (!make_a_map(&tmA, Ab, M, K)) {
    set_error("qg_gemm_q4_0: could not encode the TMA descriptor of A");
    return QG_ERR_CUDA;
  }
  const bool w32 = aligned(blocks, 4);
  if (N % 256 == 0) {
    if (w32) gq4_launch_mt<256, true>(tmA, blocks, bias, C, M, N, K, err, s);
    else gq4_launch_mt<256, false>(tmA, blocks, bias, C, M, N, K, err, s);
  } else {
    if (w32) gq4_launch_mt<128, true>(tmA, blocks, bias, C, M, N, K, err, s);
    else gq4_launch_mt<128, false>(tmA, blocks, bias, C, M, N, K, err, s);
  }
  return check_launch("qg_gemm_q4_0");
}

extern "C" qg_status qg_gemm_q4_0_error(int M, int K, const void* ws, unsigned* code,
                                        void* stream) {
  clear_error();
  QG_REQUIRE(ws && code && M > 0 && K > 0, QG_ERR_INVALID_ARGUMENT,
             "qg_gemm_q4_0_error: null ws or code, or empty shape");
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemcpyAsync(code, reinterpret_cast<const uint8_t*>(ws) + a_bytes(M, K),
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
