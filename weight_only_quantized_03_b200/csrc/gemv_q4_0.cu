// Q4_0 dequant GEMV on the CUDA cores.
//
// Format (fuel-transformers 0.19.1, src/models/lazy_quantized_whisper.rs,
// quantize_in_out_to_q4_0, ggml BlockQ4_0): row r is K/32 blocks of 18
// bytes, an fp16 d then 16 bytes whose low nibbles are codes 0..15 and high
// nibbles codes 16..31; w = d * (n - 8). The linear is q_linear's
// y = x W^T (+ bias).
//
// Work split: a warp owns R rows; lane j takes block columns j, j+32, ...
// and, for each, the same block of all R rows, so the 32 x values of a block
// are loaded once and used R times. Per block the sum
// sum_j (n_j - 8) x_j is formed in fp32 and scaled by d once.
#include <cuda_fp16.h>

#include "qg_internal.cuh"

namespace qg {

constexpr int kQ4Warps = 8;

struct Q4Block {
  float d;
  uint32_t q[4];  // 16 nibble bytes
};

__device__ __forceinline__ Q4Block load_q4_block(const uint8_t* p) {
  // 18-byte blocks are 2-byte aligned: read nine 16-bit words.
  const uint16_t* h = reinterpret_cast<const uint16_t*>(p);
  Q4Block b;
  b.d = __half2float(__ushort_as_half(__ldg(h)));
#pragma unroll
  for (int i = 0; i < 4; ++i)
    b.q[i] = (uint32_t)__ldg(h + 1 + 2 * i) | ((uint32_t)__ldg(h + 2 + 2 * i) << 16);
  return b;
}

// (n - 8) for the nibble at bit offset `sh` of word w, exact in fp32.
__device__ __forceinline__ float nib(uint32_t w, int sh) {
  return __uint_as_float(0x4B000000u | ((w >> sh) & 0xFu)) - 8388616.0f;
}

__device__ __forceinline__ float q4_dot(const Q4Block& b, const float (&xv)[32]) {
  float p = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      p = fmaf(nib(b.q[i], 8 * k), xv[4 * i + k], p);           // code 4i+k
      p = fmaf(nib(b.q[i], 8 * k + 4), xv[16 + 4 * i + k], p);  // code 16+4i+k
    }
  }
  return p;
}

template <int NB, int R>
__global__ void __launch_bounds__(kQ4Warps * 32)
gemv_q4_0_kernel(const uint8_t* __restrict__ blocks, const float* __restrict__ x,
                 const float* __restrict__ bias, float* __restrict__ y, int N, int K, int B) {
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = (blockIdx.x * kQ4Warps + warp) * R;
  if (row0 >= N) return;
  const int nb = K >> 5;
  const size_t rowbytes = (size_t)nb * 18;
  float acc[R][NB];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int b = 0; b < NB; ++b) acc[r][b] = 0.f;

  for (int j = lane; j < nb; j += 32) {
    Q4Block blk[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int row = min(row0 + r, N - 1);
      blk[r] = load_q4_block(blocks + row * rowbytes + (size_t)j * 18);
    }
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      if (b < B) {
        float xv[32];
        const float4* xp = reinterpret_cast<const float4*>(x + (size_t)b * K + 32 * j);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float4 t = __ldg(xp + i);
          xv[4 * i] = t.x; xv[4 * i + 1] = t.y; xv[4 * i + 2] = t.z; xv[4 * i + 3] = t.w;
        }
#pragma unroll
        for (int r = 0; r < R; ++r) acc[r][b] = fmaf(blk[r].d, q4_dot(blk[r], xv), acc[r][b]);
      }
    }
  }
  pdl_trigger();
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int b = 0; b < NB; ++b) acc[r][b] = warp_sum(acc[r][b]);
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const int row = row0 + r;
      if (lane == ((r * NB + b) & 31) && row < N && b < B)
        y[(size_t)b * N + row] = acc[r][b] + (bias ? bias[row] : 0.f);
    }
}

// Staged variant (rows 16-byte aligned: K % 256 == 0 and an aligned base):
// the CTA's 8*R rows are copied to shared memory first with coalesced
// 16-byte streaming loads, all in flight at once and issued before waiting
// for the previous kernel (weights never depend on it); then each warp forms
// its R rows from shared memory exactly as above.
template <int NB, int R>
__global__ void __launch_bounds__(kQ4Warps * 32)
gemv_q4_0_staged_kernel(const uint8_t* __restrict__ blocks, const float* __restrict__ x,
                        const float* __restrict__ bias, float* __restrict__ y, int N, int K, int B) {
  extern __shared__ __align__(16) uint8_t tile[];
  constexpr int RT = kQ4Warps * R;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r0 = blockIdx.x * RT;
  const int nrows = min(RT, N - r0);
  const int nb = K >> 5;
  const size_t rowbytes = (size_t)nb * 18;
  const uint64_t pol = l2_evict_first_policy();
  const uint4* src = reinterpret_cast<const uint4*>(blocks + (size_t)r0 * rowbytes);
  uint4* dst = reinterpret_cast<uint4*>(tile);
  const int n16 = (int)((size_t)nrows * rowbytes / 16);
  for (int base = threadIdx.x; base < n16; base += blockDim.x * 8) {
    uint4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = base + u * blockDim.x;
      if (i < n16) v[u] = ld_stream_u4(src + i, pol);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = base + u * blockDim.x;
      if (i < n16) dst[i] = v[u];
    }
  }
  // the next kernel may launch now and start its own weight loads (its wait
  // still covers all of this one)
  pdl_trigger();
  __syncthreads();
  pdl_wait();  // x and bias may be written by the previous kernel
  float acc[R][NB];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int b = 0; b < NB; ++b) acc[r][b] = 0.f;
  for (int j = lane; j < nb; j += 32) {
    Q4Block blk[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int lr = min(warp * R + r, nrows - 1);
      const uint16_t* h = reinterpret_cast<const uint16_t*>(tile + lr * rowbytes + (size_t)j * 18);
      blk[r].d = __half2float(__ushort_as_half(h[0]));
#pragma unroll
      for (int i = 0; i < 4; ++i) blk[r].q[i] = (uint32_t)h[1 + 2 * i] | ((uint32_t)h[2 + 2 * i] << 16);
    }
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      if (b < B) {
        float xv[32];
        const float4* xp = reinterpret_cast<const float4*>(x + (size_t)b * K + 32 * j);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float4 t = __ldg(xp + i);
          xv[4 * i] = t.x; xv[4 * i + 1] = t.y; xv[4 * i + 2] = t.z; xv[4 * i + 3] = t.w;
        }
#pragma unroll
        for (int r = 0; r < R; ++r) acc[r][b] = fmaf(blk[r].d, q4_dot(blk[r], xv), acc[r][b]);
      }
    }
  }
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int b = 0; b < NB; ++b) acc[r][b] = warp_sum(acc[r][b]);
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const int row = r0 + warp * R + r;
      if (lane == ((r * NB + b) & 31) && warp * R + r < nrows && b < B)
        y[(size_t)b * N + row] = acc[r][b] + (bias ? bias[row] : 0.f);
    }
}

constexpr size_t kQ4StagedSmem = 96 * 1024;

template <int NB, int R>
static cudaError_t q4_staged_launch_r(const uint8_t* blocks, const float* x, const float* bias,
                                      float* y, int N, int K, int B, cudaStream_t st, bool pdl) {
  ensure_smem((const void*)gemv_q4_0_staged_kernel<NB, R>, (int)kQ4StagedSmem);
  constexpr int RT = kQ4Warps * R;
  const size_t smem = (size_t)RT * (K / 32) * 18;
  return launch_pdl(gemv_q4_0_staged_kernel<NB, R>, dim3((N + RT - 1) / RT),
                    dim3(kQ4Warps * 32), smem, st, pdl, blocks, x, bias, y, N, K, B);
}

// rows per warp: as many as keep about one CTA per SM busy and the tile in
// shared memory
template <int NB>
static cudaError_t q4_staged_launch(const uint8_t* blocks, const float* x, const float* bias,
                                    float* y, int N, int K, int B, cudaStream_t st, bool pdl) {
  const size_t rowbytes = (size_t)(K / 32) * 18;
  const int sms = num_sms();
  if ((long long)N >= 4LL * kQ4Warps * sms && 4 * kQ4Warps * rowbytes <= kQ4StagedSmem)
    return q4_staged_launch_r<NB, 4>(blocks, x, bias, y, N, K, B, st, pdl);
  if ((long long)N >= 2LL * kQ4Warps * sms && 2 * kQ4Warps * rowbytes <= kQ4StagedSmem)
    return q4_staged_launch_r<NB, 2>(blocks, x, bias, y, N, K, B, st, pdl);
  return q4_staged_launch_r<NB, 1>(blocks, x, bias, y, N, K, B, st, pdl);
}

template <int NB>
static cudaError_t q4_launch(const uint8_t* blocks, const float* x, const float* bias, float* y,
                             int N, int K, int B, cudaStream_t st, bool pdl) {
  if (K % 256 == 0 && aligned(blocks, 16) && (size_t)kQ4Warps * (K / 32) * 18 <= kQ4StagedSmem)
    return q4_staged_launch<NB>(blocks, x, bias, y, N, K, B, st, pdl);
  const int R = 4;
  const int grid = (N + kQ4Warps * R - 1) / (kQ4Warps * R);
  return launch_pdl(gemv_q4_0_kernel<NB, R>, dim3(grid), dim3(kQ4Warps * 32), 0, st, pdl, blocks,
                    x, bias, y, N, K, B);
}

cudaError_t gemv_q4_0_launch(const uint8_t* blocks, const float* x, const float* bias, float* y,
                             int N, int K, int B, cudaStream_t st, bool pdl) {
  for (int b0 = 0; b0 < B; b0 += 8) {
    const int nb = B - b0 < 8 ? B - b0 : 8;
    const float* xb = x + (size_t)b0 * K;
    float* yb = y + (size_t)b0 * N;
    cudaError_t e;
    if (nb == 1) e = q4_launch<1>(blocks, xb, bias, yb, N, K, nb, st, pdl);
    else if (nb == 2) e = q4_launch<2>(blocks, xb, bias, yb, N, K, nb, st, pdl);
    else if (nb <= 4) e = q4_launch<4>(blocks, xb, bias, yb, N, K, nb, st, pdl);
    else e = q4_launch<8>(blocks, xb, bias, yb, N, K, nb, st, pdl);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

__global__ void dequant_q4_0_kernel(const uint8_t* blocks, float* out, int N, int K) {
  const size_t n = (size_t)N * K;
  const int nb = K / 32;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    const size_t r = i / K;
    const int c = (int)(i % K), blk = c / 32, j = c % 32;
    const uint8_t* p = blocks + (r * nb + blk) * 18;
    const float d = __half2float(__ushort_as_half((uint16_t)(p[0] | (p[1] << 8))));
    const uint8_t byte = p[2 + (j & 15)];
    const int code = j < 16 ? (byte & 0xF) : (byte >> 4);
    out[i] = d * (float)(code - 8);
  }
}

}  // namespace qg

using namespace qg;

extern "C" qg_status qg_gemv_q4_0(const uint8_t* blocks, const float* x, const float* bias, float* y,
                                  int N, int K, int B, void* stream) {
  clear_error();
  QG_REQUIRE(N >= 0, QG_ERR_UNSUPPORTED_SHAPE, "qg_gemv_q4_0: N=%d must be >= 0", N);
  QG_REQUIRE(K >= 0 && K % 32 == 0, QG_ERR_UNSUPPORTED_SHAPE,
             "qg_gemv_q4_0: K=%d must be a non-negative multiple of 32", K);
  QG_REQUIRE(B >= 0 && B <= 32, QG_ERR_UNSUPPORTED_SHAPE, "qg_gemv_q4_0: B=%d must be in [0, 32]", B);
  if (N == 0 || B == 0) return QG_OK;
  QG_REQUIRE(blocks && x && y, QG_ERR_INVALID_ARGUMENT, "qg_gemv_q4_0: null blocks, x or y");
  QG_REQUIRE(aligned(blocks, 2), QG_ERR_MISALIGNED, "qg_gemv_q4_0: blocks not 2-byte aligned");
  QG_REQUIRE(aligned(x, 16), QG_ERR_MISALIGNED, "qg_gemv_q4_0: x not 16-byte aligned");
  QG_REQUIRE(aligned(y, 4) && (!bias || aligned(bias, 4)), QG_ERR_MISALIGNED,
             "qg_gemv_q4_0: y or bias misaligned");
  QG_REQUIRE((long long)N * K < (1LL << 40), QG_ERR_UNSUPPORTED_SHAPE, "qg_gemv_q4_0: N*K too large");
  // PDL: the kernel may start (and stage its weights) while the stream's
  // previous kernel drains; it waits for that kernel before reading x or bias
  gemv_q4_0_launch(blocks, x, bias, y, N, K, B, (cudaStream_t)stream, true);
  return check_launch("qg_gemv_q4_0");
}

extern "C" qg_status qg_dequant_q4_0(const uint8_t* blocks, float* out, int N, int K, void* stream) {
  clear_error();
  QG_REQUIRE(N >= 0 && K >= 0 && K % 32 == 0, QG_ERR_UNSUPPORTED_SHAPE,
             "qg_dequant_q4_0: N=%d K=%d (K must be a multiple of 32)", N, K);
  if ((size_t)N * K == 0) return QG_OK;
  QG_REQUIRE(blocks && out, QG_ERR_INVALID_ARGUMENT, "qg_dequant_q4_0: null blocks or out");
  launch_pdl(dequant_q4_0_kernel, dim3(num_sms() * 4), dim3(256), 0, (cudaStream_t)stream, false, blocks, out, N, K);
  return check_launch("qg_dequant_q4_0");
}
