// RMSNorm (plain and per-head), NeoX RoPE, SiLU-mul, residual add and the
// tied-embedding row dequantization.
//
// Definitions: turbospark-runtime 0.3.0, src/qwen3_asr_metal.rs, `step`
// (encode_rms_norm_bf16w[_perhead], encode_rope_neox_subdim,
// encode_silu_mul, encode_residual_add, embed_row_bytes); makima
// src/tts/qwen3/model.rs (RotaryEmbedding, apply_head_norm, Qwen3Mlp).
#include "qg_internal.cuh"

namespace qg {

// ------------------------------------------------------------- RMSNorm ---

// One CTA per row: y = x / sqrt(mean(x^2) + eps) * w.
__global__ void __launch_bounds__(256)
rmsnorm_kernel(const float* __restrict__ x, const uint16_t* __restrict__ w, float eps,
               void* __restrict__ y, int y_bf16, int dim) {
  pdl_wait();
  const int row = blockIdx.x;
  const float* xr = x + (size_t)row * dim;
  float ss = 0.f;
  for (int i = threadIdx.x * 4; i < dim; i += blockDim.x * 4) {
    const float4 v = *reinterpret_cast<const float4*>(xr + i);
    ss = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, ss))));
  }
  __shared__ float red[32];
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float t = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    t = warp_sum(t);
    if (threadIdx.x == 0) red[0] = t;
  }
  __syncthreads();
  const float inv = 1.0f / sqrtf(red[0] / (float)dim + eps);
  pdl_trigger();
  for (int i = threadIdx.x * 4; i < dim; i += blockDim.x * 4) {
    const float4 v = *reinterpret_cast<const float4*>(xr + i);
    const float o[4] = {v.x * inv * bf16_bits_to_f32(w[i]), v.y * inv * bf16_bits_to_f32(w[i + 1]),
                        v.z * inv * bf16_bits_to_f32(w[i + 2]),
                        v.w * inv * bf16_bits_to_f32(w[i + 3])};
    if (y_bf16) {
      uint16_t* yr = reinterpret_cast<uint16_t*>(y) + (size_t)row * dim + i;
      uint2 pk;
      pk.x = (uint32_t)f32_to_bf16_bits(o[0]) | ((uint32_t)f32_to_bf16_bits(o[1]) << 16);
      pk.y = (uint32_t)f32_to_bf16_bits(o[2]) | ((uint32_t)f32_to_bf16_bits(o[3]) << 16);
      *reinterpret_cast<uint2*>(yr) = pk;
    } else {
      float* yr = reinterpret_cast<float*>(y) + (size_t)row * dim + i;
      *reinterpret_cast<float4*>(yr) = make_float4(o[0], o[1], o[2], o[3]);
    }
  }
}

cudaError_t rmsnorm_launch(const float* x, const uint16_t* w, float eps, void* y, bool y_bf16,
                           int rows, int dim, cudaStream_t st, bool pdl) {
  if (rows == 0) return cudaSuccess;
  const int threads = dim >= 1024 ? 256 : 128;
  return launch_pdl(rmsnorm_kernel, dim3(rows), dim3(threads), 0, st, pdl, x, w, eps, y,
                    (int)y_bf16, dim);
}

// Per-head RMSNorm: one warp per (row, head) slice of D values.
__global__ void rmsnorm_perhead_kernel(const void* __restrict__ x, int x_bf16,
                                       const uint16_t* __restrict__ w, float eps,
                                       void* __restrict__ y, int y_bf16, int nslices, int D) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= nslices) return;
  const size_t base = (size_t)warp * D;
  float v[32];  // D <= 1024
  const int per = D >> 5;
  float ss = 0.f;
  for (int k = 0; k < per; ++k) {
    const size_t i = base + k * 32 + lane;
    const float t = x_bf16 ? bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(x)[i])
                           : reinterpret_cast<const float*>(x)[i];
    v[k] = t;
    ss = fmaf(t, t, ss);
  }
  ss = warp_sum(ss);
  const float inv = 1.0f / sqrtf(ss / (float)D + eps);
  for (int k = 0; k < per; ++k) {
    const int d = k * 32 + lane;
    const float o = v[k] * inv * bf16_bits_to_f32(w[d]);
    if (y_bf16)
      reinterpret_cast<uint16_t*>(y)[base + d] = f32_to_bf16_bits(o);
    else
      reinterpret_cast<float*>(y)[base + d] = o;
  }
}

// ---------------------------------------------------------------- RoPE ---

// Angle of pair i at position pos: pos * theta^(-2i/rd), in float64.
__device__ __forceinline__ void rope_cos_sin(int pos, int i, int rd, double theta, float& c,
                                             float& s) {
  const double inv_freq = pow(theta, -2.0 * (double)i / (double)rd);
  double sd, cd;
  sincos((double)pos * inv_freq, &sd, &cd);
  c = (float)cd;
  s = (float)sd;
}

// One thread per rotated pair (row, head, i < rd/2).
__global__ void rope_neox_kernel(void* __restrict__ x, int bf16, const int32_t* __restrict__ pos,
                                 double theta, int rows, int heads, int D, int rd) {
  const int half = rd >> 1;
  const size_t n = (size_t)rows * heads * half;
  for (size_t t = blockIdx.x * (size_t)blockDim.x + threadIdx.x; t < n;
       t += (size_t)gridDim.x * blockDim.x) {
    const int i = (int)(t % half);
    const size_t rh = t / half;
    const int row = (int)(rh / heads);
    float c, s;
    rope_cos_sin(pos[row], i, rd, theta, c, s);
    const size_t a = rh * D + i, b = a + half;
    if (bf16) {
      uint16_t* p = reinterpret_cast<uint16_t*>(x);
      const float x1 = bf16_bits_to_f32(p[a]), x2 = bf16_bits_to_f32(p[b]);
      p[a] = f32_to_bf16_bits(x1 * c - x2 * s);
      p[b] = f32_to_bf16_bits(x2 * c + x1 * s);
    } else {
      float* p = reinterpret_cast<float*>(x);
      const float x1 = p[a], x2 = p[b];
      p[a] = x1 * c - x2 * s;
      p[b] = x2 * c + x1 * s;
    }
  }
}

// ------------------------------------------------- SiLU-mul / residual ---

__global__ void silu_mul_kernel(const float* __restrict__ g, const float* __restrict__ u,
                                void* __restrict__ out, int bf16, int n) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const float z = g[i];
    const float v = z / (1.0f + expf(-z)) * u[i];
    if (bf16)
      reinterpret_cast<uint16_t*>(out)[i] = f32_to_bf16_bits(v);
    else
      reinterpret_cast<float*>(out)[i] = v;
  }
}

__global__ void residual_add_kernel(float* __restrict__ x, const float* __restrict__ d, int n) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
    x[i] += d[i];
}

// --------------------------------------------------------- embedding -----

// One CTA per sequence: x[b][c] = q * s + beta of row tokens[b].
__global__ void embed_affine8_kernel(const uint32_t* __restrict__ w, const uint16_t* __restrict__ s,
                                     const uint16_t* __restrict__ bi,
                                     const int32_t* __restrict__ tokens, float* __restrict__ x,
                                     int vocab, int hidden) {
  const int b = blockIdx.x;
  const int t = tokens[b];
  float* xr = x + (size_t)b * hidden;
  const bool ok = t >= 0 && t < vocab;
  for (int c = threadIdx.x; c < hidden; c += blockDim.x) {
    if (!ok) {
      xr[c] = __int_as_float(0x7fc00000);
      continue;
    }
    const uint32_t word = w[(size_t)t * (hidden / 4) + c / 4];
    const float q = (float)((word >> (8 * (c % 4))) & 0xFFu);
    const size_t g = (size_t)t * (hidden / 64) + c / 64;
    xr[c] = fmaf(q, bf16_bits_to_f32(s[g]), bf16_bits_to_f32(bi[g]));
  }
}

static int grid_for(size_t n, int threads) {
  size_t g = (n + threads - 1) / threads;
  const size_t cap = (size_t)num_sms() * 8;
  return (int)(g < cap ? (g > 0 ? g : 1) : cap);
}

}  // namespace qg

using namespace qg;

extern "C" qg_status qg_rmsnorm(const float* x, const uint16_t* w, float eps, void* y,
                                qg_dtype y_dtype, int rows, int dim, void* stream) {
  clear_error();
  QG_REQUIRE(rows >= 0, QG_ERR_UNSUPPORTED_SHAPE, "qg_rmsnorm: rows=%d must be >= 0", rows);
  QG_REQUIRE(dim >= 1 && dim <= 65536 && dim % 4 == 0, QG_ERR_UNSUPPORTED_SHAPE,
             "qg_rmsnorm: dim=%d must be in [1, 65536] and a multiple of 4", dim);
  QG_REQUIRE(y_dtype == QG_F32 || y_dtype == QG_BF16, QG_ERR_INVALID_ARGUMENT,
             "qg_rmsnorm: y_dtype=%d is not QG_F32 or QG_BF16", (int)y_dtype);
  QG_REQUIRE(eps >= 0.f, QG_ERR_INVALID_ARGUMENT, "qg_rmsnorm: eps must be >= 0");
  if (rows == 0) return QG_OK;
  QG_REQUIRE(x && w && y, QG_ERR_INVALID_ARGUMENT, "qg_rmsnorm: null x, w or y");
  QG_REQUIRE(aligned(x, 16) && aligned(y, y_dtype == QG_F32 ? 16 : 8), QG_ERR_MISALIGNED,
             "qg_rmsnorm: x or y is not 16-byte aligned");
  QG_REQUIRE(aligned(w, 2), QG_ERR_MISALIGNED, "qg_rmsnorm: w is not 2-byte aligned");
  rmsnorm_launch(x, w, eps, y, y_dtype == QG_BF16, rows, dim, (cudaStream_t)stream, false);
  return check_launch("qg_rmsnorm");
}

extern "C" qg_status qg_rmsnorm_perhead(const void* x, qg_dtype x_dtype, const uint16_t* w,
                                        float eps, void* y, qg_dtype y_dtype, int rows, int heads,
                                        int D, void* stream) {
  clear_error();
  QG_REQUIRE(rows >= 0 && heads >= 0, QG_ERR_UNSUPPORTED_SHAPE,
             "qg_rmsnorm_perhead: rows=%d heads=%d must be >= 0", rows, heads);
  QG_REQUIRE(D >= 32 && D <= 1024 && D % 32 == 0, QG_ERR_UNSUPPORTED_SHAPE,
             "qg_rmsnorm_perhead: D=%d must be a multiple of 32 in [32, 1024]", D);
  QG_REQUIRE((x_dtype == QG_F32 || x_dtype == QG_BF16) && (y_dtype == QG_F32 || y_dtype == QG_BF16),
             QG_ERR_INVALID_ARGUMENT, "qg_rmsnorm_perhead: bad x_dtype or y_dtype");
  QG_REQUIRE(eps >= 0.f, QG_ERR_INVALID_ARGUMENT, "qg_rmsnorm_perhead: eps must be >= 0");
  const long long ns = (long long)rows * heads;
  if (ns == 0) return QG_OK;
  QG_REQUIRE(x && w && y, QG_ERR_INVALID_ARGUMENT, "qg_rmsnorm_perhead: null x, w or y");
  QG_REQUIRE(aligned(x, x_dtype == QG_F32 ? 4 : 2) && aligned(y, y_dtype == QG_F32 ? 4 : 2) &&
                 aligned(w, 2),
             QG_ERR_MISALIGNED, "qg_rmsnorm_perhead: misaligned x, y or w");
  const int threads = 256;
  const long long blocks = (ns * 32 + threads - 1) / threads;
  QG_REQUIRE(blocks < (1LL << 31), QG_ERR_UNSUPPORTED_SHAPE, "qg_rmsnorm_perhead: too many slices");
  launch_pdl(rmsnorm_perhead_kernel, dim3((int)blocks), dim3(threads), 0, (cudaStream_t)stream, false, 
      x, x_dtype == QG_BF16, w, eps, y, y_dtype == QG_BF16, (int)ns, D);
  return check_launch("qg_rmsnorm_perhead");
}

extern "C" qg_status qg_rope_neox(void* x, qg_dtype dtype, const int32_t* pos, double theta,
                                  int rows, int heads, int D, int rotary_dim, void* stream) {
  clear_error();
  QG_REQUIRE(rows >= 0 && heads >= 0, QG_ERR_UNSUPPORTED_SHAPE,
             "qg_rope_neox: rows=%d heads=%d must be >= 0", rows, heads);
  QG_REQUIRE(D >= 2 && D % 2 == 0, QG_ERR_UNSUPPORTED_SHAPE, "qg_rope_neox: D=%d must be even", D);
  QG_REQUIRE(rotary_dim >= 2 && rotary_dim <= D && rotary_dim % 2 == 0, QG_ERR_UNSUPPORTED_SHAPE,
             "qg_rope_neox: rotary_dim=%d must be even and in [2, D]", rotary_dim);
  QG_REQUIRE(dtype == QG_F32 || dtype == QG_BF16, QG_ERR_INVALID_ARGUMENT,
             "qg_rope_neox: dtype=%d is not QG_F32 or QG_BF16", (int)dtype);
  QG_REQUIRE(theta > 0.0, QG_ERR_INVALID_ARGUMENT, "qg_rope_neox: theta must be > 0");
  if ((long long)rows * heads == 0) return QG_OK;
  QG_REQUIRE(x && pos, QG_ERR_INVALID_ARGUMENT, "qg_rope_neox: null x or pos");
  QG_REQUIRE(aligned(x, dtype == QG_F32 ? 4 : 2) && aligned(pos, 4), QG_ERR_MISALIGNED,
             "qg_rope_neox: misaligned x or pos");
  const size_t n = (size_t)rows * heads * (rotary_dim / 2);
  launch_pdl(rope_neox_kernel, dim3(grid_for(n, 256)), dim3(256), 0, (cudaStream_t)stream, false, 
      x, dtype == QG_BF16, pos, theta, rows, heads, D, rotary_dim);
  return check_launch("qg_rope_neox");
}

extern "C" qg_status qg_silu_mul(const float* gate, const float* up, void* out, qg_dtype out_dtype,
                                 int n, void* stream) {
  clear_error();
  QG_REQUIRE(n >= 0, QG_ERR_UNSUPPORTED_SHAPE, "qg_silu_mul: n=%d must be >= 0", n);
  QG_REQUIRE(out_dtype == QG_F32 || out_dtype == QG_BF16, QG_ERR_INVALID_ARGUMENT,
             "qg_silu_mul: out_dtype=%d is not QG_F32 or QG_BF16", (int)out_dtype);
  if (n == 0) return QG_OK;
  QG_REQUIRE(gate && up && out, QG_ERR_INVALID_ARGUMENT, "qg_silu_mul: null gate, up or out");
  QG_REQUIRE(aligned(gate, 4) && aligned(up, 4) && aligned(out, out_dtype == QG_F32 ? 4 : 2),
             QG_ERR_MISALIGNED, "qg_silu_mul: misaligned gate, up or out");
  launch_pdl(silu_mul_kernel, dim3(grid_for(n, 256)), dim3(256), 0, (cudaStream_t)stream, false, gate, up, out,
                                                                      out_dtype == QG_BF16, n);
  return check_launch("qg_silu_mul");
}

extern "C" qg_status qg_residual_add(float* x, const float* delta, int n, void* stream) {
  clear_error();
  QG_REQUIRE(n >= 0, QG_ERR_UNSUPPORTED_SHAPE, "qg_residual_add: n=%d must be >= 0", n);
  if (n == 0) return QG_OK;
  QG_REQUIRE(x && delta, QG_ERR_INVALID_ARGUMENT, "qg_residual_add: null x or delta");
  QG_REQUIRE(aligned(x, 4) && aligned(delta, 4), QG_ERR_MISALIGNED,
             "qg_residual_add: misaligned x or delta");
  launch_pdl(residual_add_kernel, dim3(grid_for(n, 256)), dim3(256), 0, (cudaStream_t)stream, false, x, delta, n);
  return check_launch("qg_residual_add");
}

extern "C" qg_status qg_embed_affine8_g64(const uint32_t* w, const uint16_t* scales,
                                          const uint16_t* biases, const int32_t* tokens, float* x,
                                          int vocab, int hidden, int B, void* stream) {
  clear_error();
  QG_REQUIRE(vocab >= 1 && hidden >= 0 && hidden % 64 == 0 && B >= 0, QG_ERR_UNSUPPORTED_SHAPE,
             "qg_embed_affine8_g64: vocab=%d hidden=%d B=%d (hidden must be a multiple of 64)",
             vocab, hidden, B);
  if (B == 0 || hidden == 0) return QG_OK;
  QG_REQUIRE(w && scales && biases && tokens && x, QG_ERR_INVALID_ARGUMENT,
             "qg_embed_affine8_g64: null pointer argument");
  QG_REQUIRE(aligned(w, 4) && aligned(tokens, 4) && aligned(x, 4) && aligned(scales, 2) &&
                 aligned(biases, 2),
             QG_ERR_MISALIGNED, "qg_embed_affine8_g64: misaligned argument");
  launch_pdl(embed_affine8_kernel, dim3(B), dim3(256), 0, (cudaStream_t)stream, false, w, scales, biases, tokens, x, vocab,
                                                            hidden);
  return check_launch("qg_embed_affine8_g64");
}
