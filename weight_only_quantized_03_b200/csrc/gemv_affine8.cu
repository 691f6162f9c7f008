// Affine-INT8 group-64 dequant GEMV on the CUDA cores.
//
// Format (turbospark-runtime 0.3.0, src/qwen3_asr_metal.rs, PackedLinear /
// load_packed_linear): row r of W is K code bytes packed four to a
// little-endian u32; group g = c / 64 of row r has a bf16 scale s and bias
// beta; the weight is q * s + beta.
//
// The kernel uses the affine factorisation of each 16-column chunk of a
// group:  sum_c (q_c s + beta) x_c = s * (sum_c q_c x_c) + beta * (sum_c x_c).
// q_c x_c is exact in fp32 when x is bf16 (8-bit by 8-bit significands), so
// the only roundings are the fp32 accumulations.
//
// Work split: a warp owns R consecutive rows; each lane streams 16-byte
// chunks (16 columns) of those rows, two chunks per loop trip, so a lane has
// 2R independent 16-byte loads in flight. Weights are read with streaming
// (L1 no-allocate, L2 evict-first) loads; x comes through the read-only
// path and stays in L1. Partial sums are reduced with warp shuffles. A
// launch may cover up to four matrices that share x (e.g. q, k and v).
#include "qg_internal.cuh"

namespace qg {

constexpr int kGemvWarps = 8;
constexpr int kMaxSegs = 4;

struct GemvParams {
  GemvSeg seg[kMaxSegs];
  int cta_start[kMaxSegs + 1];
  int nseg;
  const void* x;
  int K;
  int B;     // batch rows handled by this launch (<= NB)
  int x_ld;  // elements between batch rows of x
};

template <bool XF32>
__device__ __forceinline__ void load_x16(const void* x, int ld, int b, int col,
                                         float (&xv)[16]) {
  if (XF32) {
    const float4* p = reinterpret_cast<const float4*>(
        reinterpret_cast<const float*>(x) + (size_t)b * ld + col);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float4 t = __ldg(p + i);
      xv[4 * i] = t.x; xv[4 * i + 1] = t.y; xv[4 * i + 2] = t.z; xv[4 * i + 3] = t.w;
    }
  } else {
    const uint4* p = reinterpret_cast<const uint4*>(
        reinterpret_cast<const uint16_t*>(x) + (size_t)b * ld + col);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      uint4 t = __ldg(p + i);
      xv[8 * i + 0] = bf16_lo(t.x); xv[8 * i + 1] = bf16_hi(t.x);
      xv[8 * i + 2] = bf16_lo(t.y); xv[8 * i + 3] = bf16_hi(t.y);
      xv[8 * i + 4] = bf16_lo(t.z); xv[8 * i + 5] = bf16_hi(t.z);
      xv[8 * i + 6] = bf16_lo(t.w); xv[8 * i + 7] = bf16_hi(t.w);
    }
  }
}

// sum_{j<16} q_j * x_j for the 16 code bytes of one chunk.
__device__ __forceinline__ float dot16(const uint4& w, const float (&xv)[16]) {
  float p = 0.f;
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    p = fmaf(byte_to_f32<0>(ws[i]), xv[4 * i + 0], p);
    p = fmaf(byte_to_f32<1>(ws[i]), xv[4 * i + 1], p);
    p = fmaf(byte_to_f32<2>(ws[i]), xv[4 * i + 2], p);
    p = fmaf(byte_to_f32<3>(ws[i]), xv[4 * i + 3], p);
  }
  return p;
}

template <int NB, int R, bool XF32>
__global__ void __launch_bounds__(kGemvWarps * 32)
gemv_affine8_kernel(const __grid_constant__ GemvParams P) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int si = 0;
#pragma unroll
  for (int i = 1; i < kMaxSegs; ++i)
    if (i < P.nseg && (int)blockIdx.x >= P.cta_start[i]) si = i;
  const GemvSeg& S = P.seg[si];
  const int row0 = (((int)blockIdx.x - P.cta_start[si]) * kGemvWarps + warp) * R;
  const int K = P.K;
  const int nchunk = K >> 4;   // 16-byte chunks per row
  const int G = K >> 6;        // groups per row
  const uint8_t* wbase = reinterpret_cast<const uint8_t*>(S.w);

  int rows[R];
#pragma unroll
  for (int r = 0; r < R; ++r) rows[r] = min(row0 + r, S.N - 1);
  const bool active = row0 < S.N;

  float acc[R][NB];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int b = 0; b < NB; ++b) acc[r][b] = 0.f;

  // Weights do not depend on the previous kernel: issue the first loads
  // before waiting on it.
  const uint64_t pol = l2_evict_first_policy();
  uint4 w0[R], w1[R];
  int c0 = lane, c1 = lane + 32;
  if (active) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const uint8_t* rp = wbase + (size_t)rows[r] * K;
      if (c0 < nchunk) w0[r] = ld_stream_u4(rp + 16 * c0, pol);
      if (c1 < nchunk) w1[r] = ld_stream_u4(rp + 16 * c1, pol);
    }
  }
  pdl_wait();

  if (active) {
    for (int base = 0; base < nchunk; base += 64) {
      c0 = base + lane;
      c1 = c0 + 32;
      uint4 n0[R], n1[R];
      const int d0 = c0 + 64, d1 = c1 + 64;
      // prefetch the next trip's chunks
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const uint8_t* rp = wbase + (size_t)rows[r] * K;
        if (d0 < nchunk) n0[r] = ld_stream_u4(rp + 16 * d0, pol);
        if (d1 < nchunk) n1[r] = ld_stream_u4(rp + 16 * d1, pol);
      }
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int c = half ? c1 : c0;
        if (c < nchunk) {
          float s[R], bb[R];
#pragma unroll
          for (int r = 0; r < R; ++r) {
            const size_t gi = (size_t)rows[r] * G + (c >> 2);
            s[r] = bf16_bits_to_f32(__ldg(S.s + gi));
            bb[r] = bf16_bits_to_f32(__ldg(S.b + gi));
          }
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            if (b < P.B) {
              float xv[16];
              load_x16<XF32>(P.x, P.x_ld, b, 16 * c, xv);
              float xs = 0.f;
#pragma unroll
              for (int j = 0; j < 16; ++j) xs += xv[j];
#pragma unroll
              for (int r = 0; r < R; ++r) {
                const float p = dot16(half ? w1[r] : w0[r], xv);
                acc[r][b] = fmaf(s[r], p, fmaf(bb[r], xs, acc[r][b]));
              }
            }
          }
        }
      }
#pragma unroll
      for (int r = 0; r < R; ++r) { w0[r] = n0[r]; w1[r] = n1[r]; }
    }
  }
  pdl_trigger();
  if (!active) return;

#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int b = 0; b < NB; ++b) acc[r][b] = warp_sum(acc[r][b]);

#pragma unroll
  for (int r = 0; r < R; ++r) {
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const int row = row0 + r;
      if (lane == ((r * NB + b) & 31) && row < S.N && b < P.B) {
        const size_t o = (size_t)b * S.N + row;
        float v = acc[r][b];
        if (S.res) v += S.res[o];
        if (S.y_bf16)
          reinterpret_cast<uint16_t*>(S.y)[o] = f32_to_bf16_bits(v);
        else
          reinterpret_cast<float*>(S.y)[o] = v;
      }
    }
  }
}

template <int NB, int R>
static cudaError_t launch_nb_r(GemvParams& P, bool xf32, cudaStream_t st, bool pdl) {
  int total = 0;
  for (int i = 0; i < P.nseg; ++i) {
    P.cta_start[i] = total;
    total += (P.seg[i].N + kGemvWarps * R - 1) / (kGemvWarps * R);
  }
  P.cta_start[P.nseg] = total;
  if (total == 0) return cudaSuccess;
  if (xf32)
    return launch_pdl(gemv_affine8_kernel<NB, R, true>, dim3(total), dim3(kGemvWarps * 32), 0,
                      st, pdl, P);
  return launch_pdl(gemv_affine8_kernel<NB, R, false>, dim3(total), dim3(kGemvWarps * 32), 0, st,
                    pdl, P);
}

template <int NB>
static cudaError_t launch_nb(GemvParams& P, bool xf32, cudaStream_t st, bool pdl) {
  // Rows per warp: enough rows for the whole machine first, then more rows
  // per warp (more loads in flight, x reused across rows) for tall matrices.
  int rows = 0;
  for (int i = 0; i < P.nseg; ++i) rows += P.seg[i].N;
  const int warps_wanted = num_sms() * 16;
  if (rows >= 4 * warps_wanted) return launch_nb_r<NB, 4>(P, xf32, st, pdl);
  if (rows >= 2 * warps_wanted) return launch_nb_r<NB, 2>(P, xf32, st, pdl);
  return launch_nb_r<NB, 1>(P, xf32, st, pdl);
}

// Past 4 batch rows, a matrix with at least a wave of 128-row tiles (the LM
// head) takes the tensor-core matmul: each weight tile is dequantized once
// for all batch rows (the GEMV would stream it once per 8 rows).
static bool gemm_takes(const GemvSeg* segs, int nseg, const void* x, int K, int B, bool x_f32) {
  if (x_f32 || B < 5 || K % 64 != 0 || nseg > 3 || !aligned(x, 16)) return false;
  long long tiles = 0;
  for (int i = 0; i < nseg; ++i) {
    if (!aligned(segs[i].w, 16)) return false;
    if (i + 1 < nseg && segs[i].N % 128 != 0) return false;  // tiles may not straddle matrices
    tiles += (segs[i].N + 127) / 128;
  }
  return tiles >= num_sms();
}

cudaError_t gemv_affine8_launch(const GemvSeg* segs, int nseg, const void* x, bool x_f32,
                                int K, int B, cudaStream_t st, bool pdl) {
  if (gemm_takes(segs, nseg, x, K, B, x_f32)) {
    A8Seg m[3];
    for (int i = 0; i < nseg; ++i)
      m[i] = A8Seg{segs[i].w, segs[i].s, segs[i].b, segs[i].y, segs[i].res, segs[i].N,
                   segs[i].y_bf16};
    return gemm_affine8_launch(m, nseg, reinterpret_cast<const uint16_t*>(x), B, K, nullptr, st,
                               pdl, nullptr);
  }
  if (gemv_tc_eligible(segs, nseg, K, B, x_f32)) return gemv_tc_launch(segs, nseg, x, K, B, st, pdl);
  const size_t esz = x_f32 ? 4 : 2;
  for (int b0 = 0; b0 < B; b0 += 8) {
    const int nb = B - b0 < 8 ? B - b0 : 8;
    GemvParams P = {};
    P.nseg = nseg;
    P.K = K;
    P.B = nb;
    P.x_ld = K;
    P.x = reinterpret_cast<const uint8_t*>(x) + (size_t)b0 * K * esz;
    for (int i = 0; i < nseg; ++i) {
      P.seg[i] = segs[i];
      const size_t ysz = segs[i].y_bf16 ? 2 : 4;
      P.seg[i].y = reinterpret_cast<uint8_t*>(segs[i].y) + (size_t)b0 * segs[i].N * ysz;
      P.seg[i].res = segs[i].res ? segs[i].res + (size_t)b0 * segs[i].N : nullptr;
    }
    cudaError_t e;
    if (nb == 1) e = launch_nb<1>(P, x_f32, st, pdl);
    else if (nb == 2) e = launch_nb<2>(P, x_f32, st, pdl);
    else if (nb <= 4) e = launch_nb<4>(P, x_f32, st, pdl);
    else e = launch_nb<8>(P, x_f32, st, pdl);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// ------------------------------------------------------------ test exports

__global__ void unpack_affine8_kernel(const uint32_t* w, const uint16_t* s, const uint16_t* b,
                                      float* out, int N, int K, int dequant) {
  const size_t n = (size_t)N * K;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    const size_t r = i / K, c = i % K;
    const uint32_t word = w[r * (K / 4) + c / 4];
    const float q = (float)((word >> (8 * (c % 4))) & 0xFFu);
    if (dequant) {
      const size_t g = r * (K / 64) + c / 64;
      out[i] = fmaf(q, bf16_bits_to_f32(s[g]), bf16_bits_to_f32(b[g]));
    } else {
      out[i] = q;
    }
  }
}

}  // namespace qg

using namespace qg;

static qg_status validate_gemv(const uint32_t* w, const uint16_t* s, const uint16_t* b,
                               const void* x, qg_dtype xd, const void* y, qg_dtype yd,
                               const float* res, int N, int K, int B) {
  QG_REQUIRE(N >= 0, QG_ERR_UNSUPPORTED_SHAPE, "qg_gemv_affine8_g64: N=%d must be >= 0", N);
  QG_REQUIRE(K >= 0 && K % 64 == 0, QG_ERR_UNSUPPORTED_SHAPE,
             "qg_gemv_affine8_g64: K=%d must be a non-negative multiple of 64", K);
  QG_REQUIRE(B >= 0 && B <= 32, QG_ERR_UNSUPPORTED_SHAPE,
             "qg_gemv_affine8_g64: B=%d must be in [0, 32]", B);
  QG_REQUIRE(xd == QG_F32 || xd == QG_BF16, QG_ERR_INVALID_ARGUMENT,
             "qg_gemv_affine8_g64: x_dtype=%d is not QG_F32 or QG_BF16", (int)xd);
  QG_REQUIRE(yd == QG_F32 || yd == QG_BF16, QG_ERR_INVALID_ARGUMENT,
             "qg_gemv_affine8_g64: y_dtype=%d is not QG_F32 or QG_BF16", (int)yd);
  if (N == 0 || B == 0) return QG_OK;
  QG_REQUIRE(w && s && b && x && y, QG_ERR_INVALID_ARGUMENT,
             "qg_gemv_affine8_g64: null pointer among w=%p scales=%p biases=%p x=%p y=%p",
             (const void*)w, (const void*)s, (const void*)b, x, y);
  QG_REQUIRE(aligned(w, 16), QG_ERR_MISALIGNED, "qg_gemv_affine8_g64: w is not 16-byte aligned");
  QG_REQUIRE(aligned(x, 16), QG_ERR_MISALIGNED, "qg_gemv_affine8_g64: x is not 16-byte aligned");
  QG_REQUIRE(aligned(s, 2) && aligned(b, 2), QG_ERR_MISALIGNED,
             "qg_gemv_affine8_g64: scales/biases are not 2-byte aligned");
  QG_REQUIRE(aligned(y, yd == QG_F32 ? 4 : 2), QG_ERR_MISALIGNED,
             "qg_gemv_affine8_g64: y is misaligned");
  QG_REQUIRE(!res || aligned(res, 4), QG_ERR_MISALIGNED,
             "qg_gemv_affine8_g64: residual is not 4-byte aligned");
  QG_REQUIRE((long long)N * (long long)K < (1LL << 40), QG_ERR_UNSUPPORTED_SHAPE,
             "qg_gemv_affine8_g64: N*K too large");
  return QG_OK;
}

extern "C" qg_status qg_gemv_affine8_g64(const uint32_t* w, const uint16_t* scales,
                                         const uint16_t* biases, const void* x,
                                         qg_dtype x_dtype, void* y, qg_dtype y_dtype,
                                         const float* residual, int N, int K, int B,
                                         void* stream) {
  clear_error();
  qg_status st = validate_gemv(w, scales, biases, x, x_dtype, y, y_dtype, residual, N, K, B);
  if (st != QG_OK || N == 0 || B == 0) return st;
  GemvSeg seg = {w, scales, biases, y, residual, N, y_dtype == QG_BF16 ? 1 : 0};
  // PDL: the kernel may start while the stream's previous kernel drains; it
  // waits for that kernel before reading x or the residual
  gemv_affine8_launch(&seg, 1, x, x_dtype == QG_F32, K, B, (cudaStream_t)stream, true);
  return check_launch("qg_gemv_affine8_g64");
}

extern "C" qg_status qg_unpack_affine8(const uint32_t* w, float* out, int N, int K,
                                       void* stream) {
  clear_error();
  QG_REQUIRE(N >= 0 && K >= 0 && K % 4 == 0, QG_ERR_UNSUPPORTED_SHAPE,
             "qg_unpack_affine8: N=%d K=%d (K must be a multiple of 4)", N, K);
  if ((size_t)N * K == 0) return QG_OK;
  QG_REQUIRE(w && out, QG_ERR_INVALID_ARGUMENT, "qg_unpack_affine8: null w or out");
  launch_pdl(unpack_affine8_kernel, dim3(num_sms() * 4), dim3(256), 0, (cudaStream_t)stream, false, w, nullptr, nullptr, out,
                                                                          N, K, 0);
  return check_launch("qg_unpack_affine8");
}

extern "C" qg_status qg_dequant_affine8_g64(const uint32_t* w, const uint16_t* scales,
                                            const uint16_t* biases, float* out, int N, int K,
                                            void* stream) {
  clear_error();
  QG_REQUIRE(N >= 0 && K >= 0 && K % 64 == 0, QG_ERR_UNSUPPORTED_SHAPE,
             "qg_dequant_affine8_g64: N=%d K=%d (K must be a multiple of 64)", N, K);
  if ((size_t)N * K == 0) return QG_OK;
  QG_REQUIRE(w && scales && biases && out, QG_ERR_INVALID_ARGUMENT,
             "qg_dequant_affine8_g64: null pointer argument");
  launch_pdl(unpack_affine8_kernel, dim3(num_sms() * 4), dim3(256), 0, (cudaStream_t)stream, false, w, scales, biases, out,
                                                                          N, K, 1);
  return check_launch("qg_dequant_affine8_g64");
}
