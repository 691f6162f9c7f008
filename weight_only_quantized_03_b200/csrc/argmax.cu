// Greedy token selection on the device: the index of the first strict
// maximum of each logits row, NaNs skipped, 0 when no value beats -inf
// (turbospark-runtime 0.3.0, src/qwen3_asr_metal.rs, `argmax`: a fold from
// -inf that replaces the best only on a strictly greater value).
//
// Each (value, index) pair maps to one 64-bit key whose unsigned order is
// the order of the fold: the high word is the value's bits made monotone
// (-0 taken as +0), the low word is ~index, so of equal values the smaller
// index has the larger key. NaNs and -inf get key 0, which every counted
// value beats, and key 0 decodes to index 0. The maximum key is therefore
// the fold's result, whatever order the partial maxima meet in: the
// reduction is deterministic without atomics.
//
// Two launches: CTAs of 256 threads take contiguous chunks of a row and
// write their chunk's maximum key; one warp per row then reduces the chunk
// keys and writes the index.
#include <algorithm>

#include "qg_internal.cuh"

namespace qg {
namespace am {

constexpr int kThreads = 256;
constexpr int kMaxChunks = 64;  // chunks per row

__device__ __forceinline__ unsigned long long key_of(float v, int i) {
  if (!(v > -INFINITY)) return 0ull;  // NaN or -inf: never the fold's choice
  uint32_t bits = __float_as_uint(v == 0.0f ? 0.0f : v);
  bits = (bits & 0x80000000u) ? ~bits : (bits | 0x80000000u);
  return ((unsigned long long)bits << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)i);
}

__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long k) {
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long other = __shfl_xor_sync(0xffffffffu, k, o);
    k = other > k ? other : k;
  }
  return k;
}

__global__ void __launch_bounds__(kThreads) argmax_chunk_kernel(const float* __restrict__ logits,
                                                                int V, int chunk,
                                                                unsigned long long* __restrict__ keys) {
  pdl_wait();
  const int b = blockIdx.y, c = blockIdx.x;
  const float* row = logits + (size_t)b * V;
  const int lo = c * chunk, hi = min(V, lo + chunk);
  unsigned long long best = 0ull;
  for (int i = lo + threadIdx.x; i < hi; i += kThreads) {
    const unsigned long long k = key_of(__ldcg(row + i), i);
    best = k > best ? k : best;
  }
  best = warp_max_u64(best);
  __shared__ unsigned long long s[kThreads / 32];
  if ((threadIdx.x & 31) == 0) s[threadIdx.x >> 5] = best;
  __syncthreads();
  if (threadIdx.x < 32) {
    unsigned long long k = threadIdx.x < kThreads / 32 ? s[threadIdx.x] : 0ull;
    k = warp_max_u64(k);
    if (threadIdx.x == 0) keys[(size_t)b * gridDim.x + c] = k;
  }
}

__global__ void argmax_final_kernel(const unsigned long long* __restrict__ keys, int nchunk,
                                    int32_t* __restrict__ out) {
  pdl_wait();
  const int b = blockIdx.x;
  unsigned long long k = 0ull;
  for (int c = threadIdx.x; c < nchunk; c += 32) {
    const unsigned long long v = __ldcg(keys + (size_t)b * nchunk + c);
    k = v > k ? v : k;
  }
  k = warp_max_u64(k);
  if (threadIdx.x == 0) out[b] = k == 0ull ? 0 : (int32_t)(0xFFFFFFFFu - (uint32_t)(k & 0xFFFFFFFFull));
}

// Chunks per row: about two CTAs per SM over all rows, chunks of at least
// 2048 values.
inline int chunks(int B, int V) {
  long long n = (2LL * num_sms() + B - 1) / B;
  n = std::min<long long>(n, (V + 2047) / 2048);
  return (int)std::max<long long>(1, std::min<long long>(n, kMaxChunks));
}

// Selected-token log-probability (turbospark-runtime 0.3.0,
// src/qwen3_asr_metal.rs: compute_selected_logprob of the greedy token; the
// page does not print it, read as the log-softmax at the token):
//   out[b] = logits[b][t] - (M + log sum_i exp(logits[b][i] - M)), M = max.
// Chunk CTAs write (max, sum of exp(x - chunk max)) over their chunk; one
// warp per row merges the chunks in order. NaN anywhere gives NaN; a token
// outside [0, V) gives NaN.
__global__ void __launch_bounds__(kThreads) lse_chunk_kernel(const float* __restrict__ logits, int V,
                                                            int chunk, float2* __restrict__ part) {
  pdl_wait();
  const int b = blockIdx.y, c = blockIdx.x;
  const float* row = logits + (size_t)b * V;
  const int lo = c * chunk, hi = min(V, lo + chunk);
  __shared__ float s_red[kThreads / 32];
  __shared__ float s_m;
  float m = -INFINITY;
  for (int i = lo + threadIdx.x; i < hi; i += kThreads) m = fmaxf(m, __ldcg(row + i));
  bool nan = false;
  for (int i = lo + threadIdx.x; i < hi; i += kThreads) nan |= __ldcg(row + i) != __ldcg(row + i);
  m = warp_max(m);
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float mm = -INFINITY;
    for (int w = 0; w < kThreads / 32; ++w) mm = fmaxf(mm, s_red[w]);
    s_m = mm;
  }
  __syncthreads();
  const float cm = s_m;
  float sum = 0.f;
  if (cm != -INFINITY)
    for (int i = lo + threadIdx.x; i < hi; i += kThreads) sum += expf(__ldcg(row + i) - cm);
  if (nan) sum = __int_as_float(0x7fc00000);
  sum = warp_sum(sum);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = sum;
  __syncthreads();
  if (threadIdx.x == 0) {
    float ss = 0.f;
    for (int w = 0; w < kThreads / 32; ++w) ss += s_red[w];
    part[(size_t)b * gridDim.x + c] = make_float2(cm, ss);
  }
}

__global__ void lse_final_kernel(const float* __restrict__ logits, int V,
                                 const float2* __restrict__ part, int nchunk,
                                 const int32_t* __restrict__ tok, float* __restrict__ out) {
  pdl_wait();
  const int b = blockIdx.x;
  if (threadIdx.x != 0) return;
  float M = -INFINITY;
  for (int c = 0; c < nchunk; ++c) M = fmaxf(M, __ldcg(&part[(size_t)b * nchunk + c].x));
  float S = 0.f;
  for (int c = 0; c < nchunk; ++c) {
    const float2 p = __ldcg(part + (size_t)b * nchunk + c);
    if (p.x != -INFINITY || p.y != p.y) S += p.y * (p.x == M ? 1.0f : expf(p.x - M));
  }
  const int t = tok[b];
  const float x = (t >= 0 && t < V) ? __ldcg(logits + (size_t)b * V + t) : __int_as_float(0x7fc00000);
  out[b] = x - (M + logf(S));
}

}  // namespace am

size_t argmax_ws_bytes(int B, int V) { return (size_t)B * am::chunks(B, V) * 8; }

cudaError_t argmax_launch(const float* logits, int B, int V, int32_t* out, void* ws,
                          cudaStream_t st, bool pdl) {
  const int n = am::chunks(B, V);
  const int chunk = (V + n - 1) / n;
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(ws);
  cudaError_t e = launch_pdl(am::argmax_chunk_kernel, dim3(n, B), dim3(am::kThreads), 0, st, pdl,
                             logits, V, chunk, keys);
  if (e != cudaSuccess) return e;
  return launch_pdl(am::argmax_final_kernel, dim3(B), dim3(32), 0, st, pdl,
                    (const unsigned long long*)keys, n, out);
}

}  // namespace qg

using namespace qg;

extern "C" size_t qg_argmax_workspace_size(int B, int V) {
  if (B <= 0 || V <= 0) return 0;
  return argmax_ws_bytes(B, V);
}

extern "C" qg_status qg_argmax_f32(const float* logits, int B, int V, int32_t* out, void* ws,
                                   size_t ws_bytes, void* stream) {
  clear_error();
  QG_REQUIRE(B >= 0 && V >= 1, QG_ERR_UNSUPPORTED_SHAPE, "qg_argmax_f32: B=%d V=%d", B, V);
  if (B == 0) return QG_OK;
  QG_REQUIRE(logits && out, QG_ERR_INVALID_ARGUMENT, "qg_argmax_f32: null logits or out");
  QG_REQUIRE(aligned(logits, 4) && aligned(out, 4), QG_ERR_MISALIGNED,
             "qg_argmax_f32: logits or out not 4-byte aligned");
  const size_t need = argmax_ws_bytes(B, V);
  QG_REQUIRE(ws && ws_bytes >= need, QG_ERR_WORKSPACE_TOO_SMALL,
             "qg_argmax_f32: workspace of %zu bytes given, %zu needed", ws_bytes, need);
  QG_REQUIRE(aligned(ws, 8), QG_ERR_MISALIGNED, "qg_argmax_f32: ws not 8-byte aligned");
  argmax_launch(logits, B, V, out, ws, (cudaStream_t)stream, false);
  return check_launch("qg_argmax_f32");
}

extern "C" size_t qg_token_logprob_workspace_size(int B, int V) {
  if (B <= 0 || V <= 0) return 0;
  return argmax_ws_bytes(B, V);
}

extern "C" qg_status qg_token_logprob(const float* logits, int B, int V, const int32_t* tokens,
                                      float* out, void* ws, size_t ws_bytes, void* stream) {
  clear_error();
  QG_REQUIRE(B >= 0 && V >= 1, QG_ERR_UNSUPPORTED_SHAPE, "qg_token_logprob: B=%d V=%d", B, V);
  if (B == 0) return QG_OK;
  QG_REQUIRE(logits && tokens && out, QG_ERR_INVALID_ARGUMENT,
             "qg_token_logprob: null logits, tokens or out");
  QG_REQUIRE(aligned(logits, 4) && aligned(tokens, 4) && aligned(out, 4), QG_ERR_MISALIGNED,
             "qg_token_logprob: logits, tokens or out not 4-byte aligned");
  const size_t need = argmax_ws_bytes(B, V);
  QG_REQUIRE(ws && ws_bytes >= need, QG_ERR_WORKSPACE_TOO_SMALL,
             "qg_token_logprob: workspace of %zu bytes given, %zu needed", ws_bytes, need);
  QG_REQUIRE(aligned(ws, 8), QG_ERR_MISALIGNED, "qg_token_logprob: ws not 8-byte aligned");
  const int n = am::chunks(B, V);
  const int chunk = (V + n - 1) / n;
  cudaStream_t st = (cudaStream_t)stream;
  float2* part = reinterpret_cast<float2*>(ws);
  launch_pdl(am::lse_chunk_kernel, dim3(n, B), dim3(am::kThreads), 0, st, true, logits, V, chunk,
             part);
  launch_pdl(am::lse_final_kernel, dim3(B), dim3(32), 0, st, true, logits, V,
             (const float2*)part, n, tokens, out);
  return check_launch("qg_token_logprob");
}

