// Affine-INT8 group-64 matmul on the tcgen05 tensor cores (sm_100a):
//
//   Y[n][r] = sum_k X[n][k] * (q[r][k] * s[r][k/64] + beta[r][k/64])  (+ R[n][r])
//
// for many rows n of bf16 activations at once: the prompt rows of a batched
// prefill and the sequences of a batched decode step. Format and arithmetic
// as the GEMV (turbospark-runtime 0.3.0, src/qwen3_asr_metal.rs,
// PackedLinear / load_packed_linear); the prompt rows of `transcribe_with_details`
// go through the same linears one row after another on the page, here all
// at once.
//
// Roles: one CTA per (128 rows of W, NT rows of X) output tile over the whole
// of K, in stages of 64 columns (one quantization group):
//   * warps 0-7 dequantize W: two threads per row, 32 codes each, with the
//     raw bytes of the next stages already in flight in registers. The weight
//     w = q * s + beta (exact product, one fp32 rounding) is split into
//     hi = bf16(w) and lo = bf16(w - hi) (w - hi is exact in fp32), both
//     stored in the K-major 128-byte-swizzled layout the tensor core reads
//     (16-byte chunk c of row r at chunk c ^ (r % 8) of its 1024-byte atom).
//     hi + lo carries w to about 2^-18 relative, so the bf16 operands lose
//     nothing the oracle keeps (x is bf16 already).
//   * warp 9 loads X's NT x 64 tile of each stage with one TMA tensor copy
//     (rows past the last are zero-filled);
//   * warp 8 allocates the tensor-memory accumulator; its lane 0 issues
//     tcgen05.mma (M = 128, N = NT, K = 16, bf16 -> fp32) twice per 16
//     columns (hi, then lo) and frees each stage with tcgen05.commit;
//   * warps 0-7 then read the accumulator (lane = row of W, column = row of
//     X) and store Y (+ R), fp32 or bf16: a warp's 32 lanes write 32
//     consecutive outputs of one X row.
// Every wait is bounded (1 s); a wait that gives up sets a CTA-wide abort
// flag and the caller's error word; tensor memory is freed only after the
// last commit has landed.
#include "qg_internal.cuh"
#include "tcgen05_util.cuh"

namespace qg {
namespace ga8 {

using namespace tc;

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kProducers = 256;            // warps 0-7: W
constexpr int kThreads = kProducers + 64;  // + warp 8 (MMA) + warp 9 (TMA for X)
constexpr int kPrefetch = 2;               // W stages in flight in registers
constexpr int kMaxSegs = 3;

struct Seg {
  const uint8_t* w;    // codes [N][K]
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
};

template <int NT>
struct Cfg {
  static constexpr int kStageA = 2 * kBM * kBK * 2;  // hi and lo: 32 KB
  static constexpr int kStageB = NT * kBK * 2;
  static constexpr int kStage = kStageA + kStageB;
  static constexpr int kStages = (200 * 1024) / kStage < 6 ? (200 * 1024) / kStage : 6;
  static constexpr int kSmem = 1024 + kStages * kStage + 1024;
  static constexpr int kTmemCols = NT < 32 ? 32 : NT;
};

__device__ __forceinline__ uint32_t bf16_bits(float v) {
  return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v));
}

// dequantize 32 codes (two uint4 of code bytes) with scale s and bias beta,
// and store hi and lo halves as 4 swizzled 16-byte chunks each
__device__ __forceinline__ void store_w32(uint8_t* hi_tile, uint8_t* lo_tile, int r, int chunk0,
                                          const uint4& c0, const uint4& c1, float s, float beta) {
  const uint32_t wd[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) {
    uint32_t hv[4], lv[4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t word = wd[2 * cc + h];
#pragma unroll
      for (int p = 0; p < 2; ++p) {
        float w2[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float q = __uint_as_float(0x4B000000u | ((word >> (8 * (2 * p + e))) & 0xFFu)) -
                          8388608.0f;
          w2[e] = fmaf(q, s, beta);
        }
        const uint32_t h0 = bf16_bits(w2[0]), h1 = bf16_bits(w2[1]);
        const float r0 = w2[0] - __uint_as_float(h0 << 16), r1 = w2[1] - __uint_as_float(h1 << 16);
        hv[2 * h + p] = h0 | (h1 << 16);
        lv[2 * h + p] = bf16_bits(r0) | (bf16_bits(r1) << 16);
      }
    }
    const int c = chunk0 + cc;
    const int off = r * 128 + ((c ^ (r & 7)) << 4);
    *reinterpret_cast<uint4*>(hi_tile + off) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
    *reinterpret_cast<uint4*>(lo_tile + off) = make_uint4(lv[0], lv[1], lv[2], lv[3]);
  }
}

__device__ __forceinline__ int seg_of(const Params& P, int tile) {
  int si = 0;
#pragma unroll
  for (int i = 1; i < kMaxSegs; ++i)
    if (i < P.nseg && tile >= P.seg[i].tile0) si = i;
  return si;
}

template <int NT>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_affine8_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ Params P,
                           unsigned* __restrict__ err) {
  using G = Cfg<NT>;
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
  const int tile = blockIdx.x, n0 = blockIdx.y * NT;
  const Seg& S = P.seg[seg_of(P, tile)];
  const int row0 = (tile - S.tile0) * kBM;
  const int K = P.K, nk = K / kBK, Kg = K / 64;

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
  // the next kernel of a chain may start its own weight loads
  pdl_trigger();

  bool ok = true;
  if (warp < 8) {
    // ------------------------------------------------------ W producers
    const int r = tid >> 1, half = tid & 1;
    const int wr = min(row0 + r, S.N - 1);  // rows past N are computed, never stored
    const uint8_t* wrow = S.w + (size_t)wr * K + 32 * half;
    const uint16_t* srow = S.s + (size_t)wr * Kg;
    const uint16_t* brow = S.b + (size_t)wr * Kg;
    uint4 raw[kPrefetch][2];
    float rs[kPrefetch], rb[kPrefetch];
    auto fetch = [&](int kb, int u) {
      const uint4* p = reinterpret_cast<const uint4*>(wrow + (size_t)kb * kBK);
      raw[u][0] = ld_nc_u4(p);
      raw[u][1] = ld_nc_u4(p + 1);
      rs[u] = bf16_bits_to_f32(__ldg(srow + kb));
      rb[u] = bf16_bits_to_f32(__ldg(brow + kb));
    };
#pragma unroll
    for (int u = 0; u < kPrefetch; ++u)
      if (u < nk) fetch(u, u);
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
        uint8_t* st = stages + (size_t)s * G::kStage;
        store_w32(st, st + kBM * kBK * 2, r, 4 * half, raw[u][0], raw[u][1], rs[u], rb[u]);
        if (kb + kPrefetch < nk) fetch(kb + kPrefetch, u);
        // make the generic-proxy stores visible to the tensor core
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_arrive(&full[s]);
      }
    }
    if (!ok) *abort = 1;
  } else if (warp == 9) {
    // ------------------------------------------------- X by TMA (lane 0)
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmX)) : "memory");
      pdl_wait();  // X is written by the previous kernel
      int issued = 0;
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % G::kStages;
        if (kb >= G::kStages &&
            !wait_bar(&empty[s], (uint32_t)((kb / G::kStages) + 1) & 1u, abort)) {
          ok = false;
          *abort = 1;
          break;
        }
        mbar_expect_tx(&tfull[s], (uint32_t)G::kStageB);
        asm volatile(
            "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
            " [%0], [%1, {%2, %3}], [%4];" ::"r"(
                smem_u32(stages + (size_t)s * G::kStage + G::kStageA)),
            "l"(reinterpret_cast<uint64_t>(&tmX)), "r"(kb * kBK), "r"(n0),
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
    const uint32_t idesc = instr_desc<NT>();
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
#pragma unroll
        for (int part = 0; part < 2; ++part) {  // hi, then lo
          const uint64_t da = smem_desc(sa + part * kBM * kBK * 2 + k * 32);
          const uint32_t acc = (kb > 0 || k > 0 || part > 0) ? 1u : 0u;
          asm volatile(
              "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
              " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem),
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
  if (warp < 8) {
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
    const bool landed = (st & 1) != 0, aborted = (st & 2) != 0;
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    pdl_wait();  // the residual is written upstream
    if (landed && !aborted) {
      // warp w reads tensor-memory lanes 32 (w % 4) .. +31 (rows of W) and
      // half of the NT columns (rows of X), 8 at a time
      const int q = warp & 3, hf = warp >> 2;
      const int r = row0 + 32 * q + lane;
#pragma unroll 1
      for (int c0 = hf * (NT / 2); c0 < (hf + 1) * (NT / 2); c0 += 8) {
        uint32_t v[8];
        const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)c0;
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
              "=r"(v[7])
            : "r"(ta));
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        if (r < S.N) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int n = n0 + c0 + j;
            if (n >= P.T) break;
            const size_t o = (size_t)n * S.N + r;
            float val = __uint_as_float(v[j]);
            if (S.res) val += S.res[o];
            if (S.y_bf16)
              reinterpret_cast<uint16_t*>(S.y)[o] = f32_to_bf16_bits(val);
            else
              reinterpret_cast<float*>(S.y)[o] = val;
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

}  // namespace ga8

// The host side shared by the public entry point, the prefill and the
// batched decode step: the segments (up to 3 matrices that share X), X bf16
// [T][K]. NT (rows of X per tile) is chosen so that the launch has about a
// wave of CTAs or more.
template <int NT>
static cudaError_t ga8_launch_nt(const CUtensorMap& map, const ga8::Params& P, int tiles,
                                 unsigned* err, cudaStream_t st, bool pdl) {
  using G = ga8::Cfg<NT>;
  ensure_smem((const void*)ga8::gemm_affine8_tc_kernel<NT>, G::kSmem);
  const dim3 grid(tiles, (P.T + NT - 1) / NT);
  return launch_pdl(ga8::gemm_affine8_tc_kernel<NT>, grid, dim3(ga8::kThreads), (size_t)G::kSmem,
                    st, pdl, map, P, err);
}

int gemm_affine8_tile_rows(int tiles_m, int T) {
  // the widest tile of X rows that still gives about a wave of CTAs
  const int sms = num_sms();
  for (int nt : {256, 128, 64, 32}) {
    if (T >= nt && (long long)tiles_m * ((T + nt - 1) / nt) >= sms) return nt;
  }
  return T > 16 ? 32 : 16;
}

cudaError_t gemm_affine8_launch(const A8Seg* segs, int nseg, const uint16_t* X, int T, int K,
                                unsigned* err, cudaStream_t st, bool pdl, int* nt_used) {
  ga8::Params P = {};
  P.nseg = nseg;
  P.T = T;
  P.K = K;
  int tiles = 0;
  for (int i = 0; i < nseg; ++i) {
    P.seg[i] = ga8::Seg{reinterpret_cast<const uint8_t*>(segs[i].w), segs[i].s, segs[i].b,
                        segs[i].y, segs[i].res, segs[i].N, segs[i].y_bf16, tiles};
    tiles += (segs[i].N + ga8::kBM - 1) / ga8::kBM;
  }
  if (tiles == 0 || T == 0) return cudaSuccess;
  // a few rows of X: the codes go to the tensor core as they are and each
  // group's scale and bias apply to its partial sums (no dequantised tile)
  if (gemm_affine8_skinny_ok(T, K) && nseg <= 3) {
    if (nt_used) *nt_used = T <= 16 ? 16 : 32;
    return gemm_affine8_skinny_launch(segs, nseg, X, T, K, err, st, pdl);
  }
  const int NT = gemm_affine8_tile_rows(tiles, T);
  if (nt_used) *nt_used = NT;
  CUtensorMap map;
  if (!make_bf16_map(&map, X, T, K, NT)) return cudaErrorInvalidValue;
  switch (NT) {
    case 256: return ga8_launch_nt<256>(map, P, tiles, err, st, pdl);
    case 128: return ga8_launch_nt<128>(map, P, tiles, err, st, pdl);
    case 64: return ga8_launch_nt<64>(map, P, tiles, err, st, pdl);
    case 32: return ga8_launch_nt<32>(map, P, tiles, err, st, pdl);
    default: return ga8_launch_nt<16>(map, P, tiles, err, st, pdl);
  }
}

}  // namespace qg

using namespace qg;

extern "C" qg_status qg_gemm_affine8_g64(const uint32_t* w, const uint16_t* scales,
                                         const uint16_t* biases, const uint16_t* x, void* y,
                                         qg_dtype y_dtype, const float* residual, int N, int K,
                                         int T, void* ws, size_t ws_bytes, void* stream) {
  clear_error();
  QG_REQUIRE(N >= 0 && K >= 0 && T >= 0, QG_ERR_UNSUPPORTED_SHAPE,
             "qg_gemm_affine8_g64: N=%d K=%d T=%d must be >= 0", N, K, T);
  QG_REQUIRE(K % 64 == 0 && K > 0, QG_ERR_UNSUPPORTED_SHAPE,
             "qg_gemm_affine8_g64: K=%d must be a positive multiple of 64", K);
  QG_REQUIRE(y_dtype == QG_F32 || y_dtype == QG_BF16, QG_ERR_INVALID_ARGUMENT,
             "qg_gemm_affine8_g64: y_dtype=%d", (int)y_dtype);
  QG_REQUIRE(!residual || y_dtype == QG_F32, QG_ERR_INVALID_ARGUMENT,
             "qg_gemm_affine8_g64: a residual needs an fp32 y");
  QG_REQUIRE((long long)T * K < (1LL << 40) && (long long)T * N < (1LL << 40) &&
                 (long long)N * K < (1LL << 40) && T < (1 << 30),
             QG_ERR_UNSUPPORTED_SHAPE, "qg_gemm_affine8_g64: too large");
  if (N == 0 || T == 0) return QG_OK;
  QG_REQUIRE(w && scales && biases && x && y, QG_ERR_INVALID_ARGUMENT,
             "qg_gemm_affine8_g64: null pointer");
  QG_REQUIRE(aligned(w, 16) && aligned(x, 16), QG_ERR_MISALIGNED,
             "qg_gemm_affine8_g64: w and x must be 16-byte aligned");
  QG_REQUIRE(aligned(scales, 2) && aligned(biases, 2) && aligned(y, 4) && aligned(residual, 4),
             QG_ERR_MISALIGNED, "qg_gemm_affine8_g64: scales/biases/y/residual misaligned");
  QG_REQUIRE(ws && ws_bytes >= 4 && aligned(ws, 4), QG_ERR_WORKSPACE_TOO_SMALL,
             "qg_gemm_affine8_g64: ws must hold the 4-byte error word");
  cudaStream_t s = (cudaStream_t)stream;
  unsigned* err = reinterpret_cast<unsigned*>(ws);
  cudaMemsetAsync(err, 0, 4, s);
  const A8Seg seg = {w, scales, biases, y, residual, N, y_dtype == QG_BF16 ? 1 : 0};
  cudaError_t e = gemm_affine8_launch(&seg, 1, x, T, K, err, s, false, nullptr);
  if (e == cudaErrorInvalidValue) {
    set_error("qg_gemm_affine8_g64: could not encode the TMA descriptor of x");
    return QG_ERR_CUDA;
  }
  return check_launch("qg_gemm_affine8_g64");
}
