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
//   2. gemm_q4_0_tc_kernel, one CTA per 128 x BN output tile:
//      * warps 0-7 (producers) fill a ring of shared-memory stages, each
//        128 rows of A and BN rows of W over 64 columns of K, in the
//        K-major 128-byte-swizzled layout the tensor core reads (16-byte
//        chunk c of row r stored at chunk c ^ (r % 8) of its 1024-byte
//        atom). W is dequantized on the way: two Q4_0 blocks per row.
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
#include <algorithm>

#include "qg_internal.cuh"

namespace qg {
namespace gq4 {

constexpr int kBM = 128;
constexpr int kBK = 64;               // one 128-byte swizzle row of bf16
constexpr int kProducers = 256;       // warps 0-7
constexpr int kThreads = kProducers + 32;
constexpr unsigned long long kWaitNs = 1000000000ull;

template <int BN>
struct Cfg {
  static constexpr int kStageA = kBM * kBK * 2;   // 16 KB
  static constexpr int kStageB = BN * kBK * 2;    // 16 or 32 KB
  static constexpr int kStage = kStageA + kStageB;
  static constexpr int kStages = BN == 256 ? 4 : 6;
  static constexpr int kSmem = 1024 + kStages * kStage + 1024;  // + align slack + barriers
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

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_q4_0_tc_kernel(const uint16_t* __restrict__ Ab, const uint8_t* __restrict__ blocks,
                        const float* __restrict__ bias, float* __restrict__ C, int M, int N, int K,
                        unsigned* __restrict__ err) {
  using G = Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* stages = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + G::kStages * G::kStage);
  uint64_t* empty = full + G::kStages;
  uint64_t* done = empty + G::kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n0 = blockIdx.x * BN, m0 = blockIdx.y * kBM;
  const int nk = K / kBK, kblocks = K / 32;

  if (tid == 0) {
    for (int s = 0; s < G::kStages; ++s) {
      mbar_init(&full[s], kProducers);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 8) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(BN));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;

  bool ok = true;
  if (warp < 8) {
    // -------------------------------------------------------- producers
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % G::kStages;
      if (kb >= G::kStages && !wait_bar(&empty[s], (uint32_t)((kb / G::kStages) + 1) & 1u, abort)) {
        ok = false;
        break;
      }
      uint8_t* sa = stages + (size_t)s * G::kStage;
      uint8_t* sb = sa + G::kStageA;
      // A: 128 rows x 8 chunks of 16 bytes
#pragma unroll
      for (int j = 0; j < (kBM * 8) / kProducers; ++j) {
        const int i = tid + j * kProducers, r = i >> 3, c = i & 7;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (m0 + r < M)
          v = __ldg(reinterpret_cast<const uint4*>(Ab + (size_t)(m0 + r) * K + kb * kBK + c * 8));
        *reinterpret_cast<uint4*>(sa + r * 128 + ((c ^ (r & 7)) << 4)) = v;
      }
      // W: BN rows x two Q4_0 blocks, dequantized to bf16
#pragma unroll
      for (int j = 0; j < (BN * 2) / kProducers; ++j) {
        const int i = tid + j * kProducers, r = i >> 1, h = i & 1;
        const uint16_t* bp = reinterpret_cast<const uint16_t*>(
            blocks + ((size_t)(n0 + r) * kblocks + (size_t)kb * 2 + h) * 18);
        uint16_t u[9];
#pragma unroll
        for (int q = 0; q < 9; ++q) u[q] = __ldg(bp + q);
        const float d = __half2float(__ushort_as_half(u[0]));
        float w[32];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const uint32_t b2 = u[1 + q];  // bytes 2q, 2q+1 of the 16 code bytes
          w[2 * q] = (float)((int)(b2 & 0xFu) - 8) * d;
          w[2 * q + 1] = (float)((int)((b2 >> 8) & 0xFu) - 8) * d;
          w[2 * q + 16] = (float)((int)((b2 >> 4) & 0xFu) - 8) * d;
          w[2 * q + 17] = (float)((int)((b2 >> 12) & 0xFu) - 8) * d;
        }
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const int c = h * 4 + cc;
          uint4 v;
          v.x = pack_bf16x2(w[cc * 8 + 0], w[cc * 8 + 1]);
          v.y = pack_bf16x2(w[cc * 8 + 2], w[cc * 8 + 3]);
          v.z = pack_bf16x2(w[cc * 8 + 4], w[cc * 8 + 5]);
          v.w = pack_bf16x2(w[cc * 8 + 6], w[cc * 8 + 7]);
          *reinterpret_cast<uint4*>(sb + r * 128 + ((c ^ (r & 7)) << 4)) = v;
        }
      }
      // make the generic-proxy stores visible to the tensor core
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(&full[s]);
    }
    if (!ok) *abort = 1;
  } else if (lane == 0) {
    // ------------------------------------------------------- MMA issuer
    const uint32_t idesc = instr_desc<BN>();
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % G::kStages;
      if (!wait_bar(&full[s], (uint32_t)(kb / G::kStages) & 1u, abort)) {
        ok = false;
        *abort = 1;
        break;
      }
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t sa = smem_u32(stages + (size_t)s * G::kStage);
      const uint32_t sb = sa + G::kStageA;
#pragma unroll
      for (int k = 0; k < kBK / 16; ++k) {
        const uint64_t da = smem_desc(sa + k * 32), db = smem_desc(sb + k * 32);
        const uint32_t acc = (kb > 0 || k > 0) ? 1u : 0u;
        asm volatile(
            "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
            " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem),
            "l"(da), "l"(db), "r"(idesc), "r"(acc)
            : "memory");
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
      const int q = warp & 3, half = warp >> 2;
      const int m = m0 + 32 * q + lane;
#pragma unroll 1
      for (int c0 = half * (BN / 2); c0 < (half + 1) * (BN / 2); c0 += 32) {
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
        if (m < M) {
          float* crow = C + (size_t)m * N + n0 + c0;
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            float4 o = make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]),
                                   __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
            if (bias) {
              o.x += bias[n0 + c0 + j];
              o.y += bias[n0 + c0 + j + 1];
              o.z += bias[n0 + c0 + j + 2];
              o.w += bias[n0 + c0 + j + 3];
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
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(BN));
  }
}

}  // namespace gq4

static size_t a_bytes(int M, int K) { return (((size_t)M * K * 2) + 255) & ~(size_t)255; }

template <int BN>
static cudaError_t gq4_launch(const uint16_t* Ab, const uint8_t* blocks, const float* bias,
                              float* C, int M, int N, int K, unsigned* err, cudaStream_t st) {
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(gq4::gemm_q4_0_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         gq4::Cfg<BN>::kSmem);
    attr = true;
  }
  dim3 grid(N / BN, (M + gq4::kBM - 1) / gq4::kBM);
  return launch_pdl(gq4::gemm_q4_0_tc_kernel<BN>, grid, dim3(gq4::kThreads),
                    (size_t)gq4::Cfg<BN>::kSmem, st, false, Ab, blocks, bias, C, M, N, K, err);
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
  if (N % 256 == 0)
    gq4_launch<256>(Ab, blocks, bias, C, M, N, K, err, s);
  else
    gq4_launch<128>(Ab, blocks, bias, C, M, N, K, err, s);
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
