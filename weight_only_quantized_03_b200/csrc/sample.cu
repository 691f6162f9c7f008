// Token sampling on the device: repetition penalty, temperature, top-k and
// a draw from the top-k softmax (makima src/tts/qwen3 `sample_token` and
// `apply_repetition_penalty`), in the page's fp32 arithmetic and order.
//
//   s_i = logits[b][i]; for every past token t of the row (each occurrence,
//       in order; t outside [0, V) skipped): s_t = s_t < 0 ? s_t * p : s_t / p
//   top_k == 0 or temperature == 0: the greedy token (the first strict
//       maximum, as qg_argmax_f32)
//   otherwise: t_i = s_i / temperature; the k largest t in descending order,
//       equal values by index (a stable sort); e_j = exp(t_j - t_0) summed in
//       order; the first j whose running sum of e_j / sum reaches r[b] is
//       drawn (j = 0 if none does).
//
// Four launches for top-k: copy + penalty; per 2048-value chunk a bitonic
// sort of order-preserving 64-bit keys (value bits made monotone, then
// ~index) in shared memory, keeping the chunk's k best; one CTA per row
// sorts the chunks' candidates, and one thread walks the k values in order.
// NaN scores are never drawn (key 0).
#include <algorithm>

#include "qg_internal.cuh"

namespace qg {
namespace sp {

constexpr int kThreads = 256;
constexpr int kChunk = 2048;       // values per chunk CTA (sorted in shared memory)
constexpr int kMaxK = 64;
constexpr int kMaxCand = 8192;     // candidates the final sort holds (power of two)

__device__ __forceinline__ unsigned long long key_of(float v, int i) {
  if (v != v) return 0ull;  // NaN: never drawn
  uint32_t bits = __float_as_uint(v == 0.0f ? 0.0f : v);
  bits = (bits & 0x80000000u) ? ~bits : (bits | 0x80000000u);
  return ((unsigned long long)bits << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)i);
}

__device__ __forceinline__ float value_of(unsigned long long k) {
  uint32_t bits = (uint32_t)(k >> 32);
  bits = (bits & 0x80000000u) ? (bits & 0x7FFFFFFFu) : ~bits;
  return __uint_as_float(bits);
}

__device__ __forceinline__ int index_of(unsigned long long k) {
  return (int)(0xFFFFFFFFu - (uint32_t)(k & 0xFFFFFFFFull));
}

// Bitonic sort of n (a power of two) keys in shared memory, descending.
__device__ void sort_desc(unsigned long long* a, int n) {
  for (int size = 2; size <= n; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      __syncthreads();
      for (int i = threadIdx.x; i < n / 2; i += blockDim.x) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool desc = (lo & size) == 0;
        const unsigned long long x = a[lo], y = a[hi];
        if ((x < y) == desc) {
          a[lo] = y;
          a[hi] = x;
        }
      }
    }
  }
  __syncthreads();
}

// s = logits, then the repetition penalty of the row's past tokens, applied
// one occurrence after another by one thread (as the page's loop).
__global__ void __launch_bounds__(kThreads) penalty_kernel(const float* __restrict__ logits, int V,
                                                          const int32_t* __restrict__ past, int P,
                                                          float penalty, float* __restrict__ s) {
  pdl_wait();
  const int b = blockIdx.x;
  const float* src = logits + (size_t)b * V;
  float* dst = s + (size_t)b * V;
  for (int i = threadIdx.x; i < V; i += kThreads) dst[i] = __ldcg(src + i);
  __syncthreads();
  if (threadIdx.x == 0 && past && penalty != 1.0f) {
    for (int j = 0; j < P; ++j) {
      const int t = past[(size_t)b * P + j];
      if (t < 0 || t >= V) continue;
      const float v = dst[t];
      dst[t] = v < 0.0f ? v * penalty : v / penalty;
    }
  }
}

// The k best keys of one chunk of row b, t = s / temperature.
__global__ void __launch_bounds__(kThreads) chunk_topk_kernel(const float* __restrict__ s, int V,
                                                             float temperature, int k,
                                                             unsigned long long* __restrict__ cand) {
  pdl_wait();
  __shared__ unsigned long long keys[kChunk];
  const int b = blockIdx.y, c = blockIdx.x;
  const float* row = s + (size_t)b * V;
  for (int i = threadIdx.x; i < kChunk; i += kThreads) {
    const int idx = c * kChunk + i;
    keys[i] = idx < V ? key_of(__ldcg(row + idx) / temperature, idx) : 0ull;
  }
  sort_desc(keys, kChunk);
  for (int j = threadIdx.x; j < k; j += kThreads)
    cand[((size_t)b * gridDim.x + c) * k + j] = keys[j];
}

// Sort the row's candidates; walk the k best in order against r[b].
__global__ void __launch_bounds__(kThreads) draw_kernel(const unsigned long long* __restrict__ cand,
                                                       int ncand, int k, const float* __restrict__ r,
                                                       int32_t* __restrict__ out) {
  pdl_wait();
  extern __shared__ unsigned long long keys[];  // [n], n = ncand rounded up to a power of two
  const int b = blockIdx.x;
  int n = 1;
  while (n < ncand) n <<= 1;
  for (int i = threadIdx.x; i < n; i += kThreads)
    keys[i] = i < ncand ? __ldcg(cand + (size_t)b * ncand + i) : 0ull;
  sort_desc(keys, n);
  if (threadIdx.x == 0) {
    int kk = 0;  // candidates that are numbers
    while (kk < k && keys[kk] != 0ull) ++kk;
    int pick = kk > 0 ? index_of(keys[0]) : 0;
    if (kk > 0) {
      const float t0 = value_of(keys[0]);
      float sum = 0.0f;
      for (int j = 0; j < kk; ++j) sum += expf(value_of(keys[j]) - t0);
      const float rb = r[b];
      float cum = 0.0f;
      for (int j = 0; j < kk; ++j) {
        cum += expf(value_of(keys[j]) - t0) / sum;
        if (cum >= rb) {
          pick = index_of(keys[j]);
          break;
        }
      }
    }
    out[b] = pick;
  }
}

inline int chunks(int V) { return (V + kChunk - 1) / kChunk; }

}  // namespace sp

static size_t a256(size_t v) { return (v + 255) & ~(size_t)255; }

// workspace: s [B][V] fp32, then the chunk candidates [B][chunks][k] (or
// the argmax keys for the greedy case)
static size_t sample_ws_bytes(int B, int V, int top_k) {
  const size_t cand = top_k > 0 ? (size_t)B * sp::chunks(V) * top_k * 8 : 0;
  return a256((size_t)B * V * 4) + std::max(a256(cand), a256(argmax_ws_bytes(B, V)));
}

}  // namespace qg

using namespace qg;

extern "C" size_t qg_sample_workspace_size(int B, int V, int top_k) {
  if (B <= 0 || V <= 0 || top_k < 0) return 0;
  return sample_ws_bytes(B, V, top_k);
}

extern "C" qg_status qg_sample(const float* logits, int B, int V, const int32_t* past, int P,
                               float penalty, float temperature, int top_k, const float* r,
                               int32_t* out, void* ws, size_t ws_bytes, void* stream) {
  clear_error();
  QG_REQUIRE(B >= 0 && V >= 1 && P >= 0, QG_ERR_UNSUPPORTED_SHAPE, "qg_sample: B=%d V=%d P=%d", B,
             V, P);
  QG_REQUIRE(top_k >= 0 && top_k <= sp::kMaxK, QG_ERR_UNSUPPORTED_SHAPE,
             "qg_sample: top_k=%d must be in [0, %d]", top_k, sp::kMaxK);
  QG_REQUIRE(penalty > 0.0f && temperature >= 0.0f, QG_ERR_INVALID_ARGUMENT,
             "qg_sample: penalty must be > 0 and temperature >= 0");
  if (B == 0) return QG_OK;
  const bool greedy = top_k == 0 || temperature == 0.0f;
  QG_REQUIRE(logits && out && (greedy || r) && (P == 0 || past), QG_ERR_INVALID_ARGUMENT,
             "qg_sample: null logits, out, r or past");
  QG_REQUIRE(aligned(logits, 4) && aligned(out, 4), QG_ERR_MISALIGNED,
             "qg_sample: logits or out not 4-byte aligned");
  const int k = greedy ? 0 : std::min(top_k, V);
  QG_REQUIRE(greedy || (size_t)sp::chunks(V) * k <= (size_t)sp::kMaxCand, QG_ERR_UNSUPPORTED_SHAPE,
             "qg_sample: V=%d with top_k=%d exceeds %d candidates", V, top_k, sp::kMaxCand);
  const size_t need = sample_ws_bytes(B, V, top_k);
  QG_REQUIRE(ws && ws_bytes >= need, QG_ERR_WORKSPACE_TOO_SMALL,
             "qg_sample: workspace of %zu bytes given, %zu needed", ws_bytes, need);
  QG_REQUIRE(aligned(ws, 256), QG_ERR_MISALIGNED, "qg_sample: ws not 256-byte aligned");
  cudaStream_t st = (cudaStream_t)stream;
  float* s = reinterpret_cast<float*>(ws);
  void* rest = reinterpret_cast<uint8_t*>(ws) + a256((size_t)B * V * 4);
  launch_pdl(sp::penalty_kernel, dim3(B), dim3(sp::kThreads), 0, st, true, logits, V, past, P,
             penalty, s);
  if (greedy) {
    argmax_launch(s, B, V, out, rest, st, true);
    return check_launch("qg_sample");
  }
  const int nc = sp::chunks(V);
  unsigned long long* cand = reinterpret_cast<unsigned long long*>(rest);
  launch_pdl(sp::chunk_topk_kernel, dim3(nc, B), dim3(sp::kThreads), 0, st, true,
             (const float*)s, V, temperature, k, cand);
  int n = 1;
  while (n < nc * k) n <<= 1;
  const size_t smem = (size_t)n * 8;
  ensure_smem((const void*)sp::draw_kernel, sp::kMaxCand * 8);
  launch_pdl(sp::draw_kernel, dim3(B), dim3(sp::kThreads), smem, st, true,
             (const unsigned long long*)cand, nc * k, k, r, out);
  return check_launch("qg_sample");
}
