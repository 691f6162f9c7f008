// Internal helpers shared by the libqg translation units (GPU side only).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stdio.h>
#include <string>

#include "qg.h"

namespace qg {

// ---------------------------------------------------------------- errors --

void set_error(const char* fmt, ...);
void clear_error();

#define QG_REQUIRE(cond, code, ...)  \
  do {                               \
    if (!(cond)) {                   \
      ::qg::set_error(__VA_ARGS__);  \
      return (code);                 \
    }                                \
  } while (0)

inline bool aligned(const void* p, size_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

qg_status check_launch(const char* what);

// ---------------------------------------------------------------- launch --

// Launch with Programmatic Dependent Launch allowed: the kernel may start
// while its predecessor on the stream drains, and must call
// pdl_wait() before touching anything the predecessor writes.
void count_launch();
// Raises `func`'s dynamic shared memory limit to `bytes` on the current
// device, once per (kernel, device).
void ensure_smem(const void* func, int bytes);

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block,
                              size_t smem, cudaStream_t stream, bool pdl,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  count_launch();
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// griddepcontrol: wait for the predecessor grid's memory to be visible /
// allow the successor grid to begin launching.
__device__ __forceinline__ void pdl_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// --------------------------------------------------------- L2 prefetch --

// Work a kernel of the decode step hands to L2 at entry for a kernel that
// runs later in the chain: byte ranges (packed weights, their scales and
// biases) and, optionally, the cached K/V rows [0, position) of every
// sequence of one layer. Prefetches are hints: they move no data the kernel
// reads and complete on their own.
constexpr int kMaxPf = 12;
struct PfRange {
  const void* p;
  unsigned long long bytes;
};
struct KvPf {
  const uint16_t* kc;  // one layer's caches [B][Hkv][cap][D], or null for none
  const uint16_t* vc;
  const int32_t* pos;  // [B]: rows [0, pos[b]) of sequence b are prefetched
  int B, Hkv, cap, D;
};
struct Prefetch {
  PfRange r[kMaxPf];
  int n;
  KvPf kv;
};

// Share `part` of `parts` of the 16-byte-aligned interior of [p, p + bytes)
// (the unaligned ends, under 16 bytes each, are left out so that no byte
// outside the range is touched), in pieces of at most 32 KB.
__device__ __forceinline__ void l2_prefetch_range(const void* p, unsigned long long bytes,
                                                  unsigned part, unsigned parts) {
  const unsigned long long a0 = ((unsigned long long)(uintptr_t)p + 15ull) & ~15ull;
  const unsigned long long a1 = ((unsigned long long)(uintptr_t)p + bytes) & ~15ull;
  if (a1 <= a0) return;
  const unsigned long long per = ((a1 - a0 + parts - 1) / parts + 15ull) & ~15ull;
  unsigned long long lo = a0 + (unsigned long long)part * per;
  const unsigned long long hi = lo + per < a1 ? lo + per : a1;
  for (; lo < hi; lo += 32768ull) {
    const unsigned sz = (unsigned)(hi - lo < 32768ull ? hi - lo : 32768ull);
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(lo), "r"(sz) : "memory");
  }
}

// Issued by one thread of each CTA (part = its CTA index among `parts`).
// The positions are inputs of the step, final before its first kernel runs.
// Issued only in a library built with QG_L2_PREFETCH: measured on the B200
// (0.6B decode step, batch 1) the hints made no kernel of the chain faster,
// since each kernel already issues its first weight loads before its
// programmatic-dependent-launch wait, and the embedding kernel's share
// (layer 0's q/k/v, 4 MB from a few SMs) cost 25 us.
__device__ __forceinline__ void issue_prefetch(const Prefetch& pf, unsigned part, unsigned parts) {
#ifndef QG_L2_PREFETCH
  return;
#endif
  for (int r = 0; r < pf.n; ++r) l2_prefetch_range(pf.r[r].p, pf.r[r].bytes, part, parts);
  if (pf.kv.kc) {
    const int ranges = 2 * pf.kv.B * pf.kv.Hkv;  // (sequence, kv head) x (K, V)
    for (int j = (int)part; j < ranges; j += (int)parts) {
      const int pair = j >> 1, b = pair / pf.kv.Hkv;
      const int rows = pf.kv.pos[b];
      if (rows <= 0 || rows > pf.kv.cap) continue;
      const uint16_t* base = ((j & 1) ? pf.kv.vc : pf.kv.kc) + (size_t)pair * pf.kv.cap * pf.kv.D;
      l2_prefetch_range(base, (unsigned long long)rows * pf.kv.D * 2, 0, 1);
    }
  }
}

// ------------------------------------------------------------ timeline --

// Per-launch timestamps for diagnosing a chain of kernels inside a CUDA
// graph (qg_timeline_begin / _end). Only a library built with QG_TIMELINE
// records; otherwise the hooks compile to nothing. Each record is filled
// with atomic maxima over the launch's CTAs (zero-initialised by the
// caller): the earliest CTA entry (stored as its bitwise complement), the
// latest return from the wait for the previous kernel, the latest exit, the
// latest CTA entry.
struct TlRec {
  unsigned long long neg_entry, wait, exit, last_entry;
};

// Host side: the record for the next launch (nullptr when not recording).
// `kind` labels the launch for qg_timeline_end.
TlRec* tl_take(int kind);
// Labels the next launches of this host thread (until changed) for tl_take.
void tl_set_kind(int kind);

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
#ifdef QG_TIMELINE
__device__ __forceinline__ void tl_entry(TlRec* r) {
  if (r && threadIdx.x == 0) {
    const unsigned long long t = global_ns();
    atomicMax(&r->neg_entry, ~t);
    atomicMax(&r->last_entry, t);
  }
}
__device__ __forceinline__ void tl_wait(TlRec* r) {
  if (r && threadIdx.x == 0) atomicMax(&r->wait, global_ns());
}
__device__ __forceinline__ void tl_exit(TlRec* r) {
  if (r && threadIdx.x == 0) atomicMax(&r->exit, global_ns());
}
#else
__device__ __forceinline__ void tl_entry(TlRec*) {}
__device__ __forceinline__ void tl_wait(TlRec*) {}
__device__ __forceinline__ void tl_exit(TlRec*) {}
#endif

// Launch kinds of the decode step (labels of the timeline records).
enum TlKind { kTlEmbed = 1, kTlQkv, kTlAttn, kTlO, kTlGateUp, kTlDown, kTlHead, kTlOther };

// ----------------------------------------------------------------- loads --

// L2 policy for data read exactly once (packed weights): evict first.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// 16-byte streaming load: not kept in L1, evict-first in L2.
__device__ __forceinline__ uint4 ld_stream_u4(const void* ptr, uint64_t pol) {
  uint4 v;
  asm volatile(
      "ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(ptr), "l"(pol));
  return v;
}

__device__ __forceinline__ uint4 ld_nc_u4(const void* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t bits16) {
  return __uint_as_float(bits16 << 16);
}
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// Byte i of a 32-bit word as an exact float: the byte is placed in the low
// mantissa bits of 2^23 and 2^23 is subtracted.
template <int I>
__device__ __forceinline__ float byte_to_f32(uint32_t w) {
  const uint32_t magic = __byte_perm(w, 0x4B000000u, 0x7440u | I);
  return __uint_as_float(magic) - 8388608.0f;
}

// codes (0,1) and (2,3) of a word as fp16 pairs of q - 128: the byte
// permute makes 1024 + q (fp16 0x6400 | q), one packed subtract of 1152
// (0x6480) centres it; both steps are exact. Centred codes keep the fp32
// partial sums of a group near sum (q - 128) x instead of carrying a
// 1024 * sum(x) term, so their rounding error is that much smaller.
__device__ __forceinline__ uint32_t centre(uint32_t h2) {
  const __half2 r = __hsub2(*reinterpret_cast<const __half2*>(&h2),
                            __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480)));
  return *reinterpret_cast<const uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t codes01(uint32_t w) {
  return centre(__byte_perm(w, 0x64646464u, 0x4140u));
}
__device__ __forceinline__ uint32_t codes23(uint32_t w) {
  return centre(__byte_perm(w, 0x64646464u, 0x4342u));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

inline int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

}  // namespace qg

// Internal launchers shared between translation units (the decode step
// composes the single-op kernels). All arguments have been validated.
namespace qg {

struct GemvSeg {           // one affine8 matrix of a multi-matrix GEMV launch
  const uint32_t* w;
  const uint16_t* s;
  const uint16_t* b;
  void* y;                 // [B][N] of y_bf16 ? bf16 : fp32
  const float* res;        // nullable fp32 [B][N]
  int N;
  int y_bf16;
};

cudaError_t gemv_affine8_launch(const GemvSeg* segs, int nseg, const void* x,
                                bool x_f32, int K, int B, cudaStream_t st,
                                bool pdl);

// tensor-core streaming path of the affine8 GEMV (gemv_affine8_tc.cu)
bool gemv_tc_eligible(const GemvSeg* segs, int nseg, int K, int B, bool x_f32);
cudaError_t gemv_tc_launch(const GemvSeg* segs, int nseg, const void* x, int K, int B,
                           cudaStream_t st, bool pdl);
// The same GEMV with its input formed in the prologue: bf16(RMSNorm(x) * w)
// of fp32 x [B][K], or bf16(silu(gate) * up) of fp32 [B][K] (eligibility as
// gemv_tc_eligible with x_f32 = false). When xout is not null the formed
// bf16 input is also written there ([B][K], by one CTA).
// `pf`, when given, is L2 prefetch work issued at kernel entry.
cudaError_t gemv_tc_launch_rmsnorm(const GemvSeg* segs, int nseg, const float* x,
                                   const uint16_t* norm_w, float eps, int K, int B,
                                   cudaStream_t st, bool pdl, uint16_t* xout = nullptr,
                                   const Prefetch* pf = nullptr);
cudaError_t gemv_tc_launch_silu_mul(const GemvSeg* segs, int nseg, const float* gate,
                                    const float* up, int K, int B, cudaStream_t st, bool pdl,
                                    uint16_t* xout = nullptr, const Prefetch* pf = nullptr);
cudaError_t gemv_tc_launch_pf(const GemvSeg* segs, int nseg, const void* x, int K, int B,
                              cudaStream_t st, bool pdl, const Prefetch* pf);
// The RMSNorm prologue on x + sum_{j < nparts} parts[b][j] (fixed order),
// parts [B][nparts][K] fp32; CTA 0 stores that sum to xsum [B][K].
cudaError_t gemv_tc_launch_rmsnorm_parts(const GemvSeg* segs, int nseg, const float* x,
                                         const float* parts, int nparts, float* xsum,
                                         const uint16_t* norm_w, float eps, int K, int B,
                                         cudaStream_t st, bool pdl, uint16_t* xout,
                                         const Prefetch* pf);

cudaError_t rmsnorm_launch(const float* x, const uint16_t* w, float eps, void* y,
                           bool y_bf16, int rows, int dim, cudaStream_t st, bool pdl);

cudaError_t attention_launch(const float* q, const uint16_t* kc, const uint16_t* vc,
                             const int32_t* kv_len, const int32_t* pos_for_len,
                             void* out, bool out_bf16, int B, int H, int Hkv, int D,
                             int cap, float scale, void* ws, cudaStream_t st, bool pdl);

// o_proj fused into the decode step's attention: W_o (codes [hidden][H*D],
// scales/biases 8-byte aligned) and the partial rows out, fp32
// [B][Hkv][hidden] (one row of partial sums per KV head's query heads).
struct OProjFuse {
  const uint32_t* w;
  const uint16_t* s;
  const uint16_t* b;
  float* part;
  int hidden;
};

// The decode step's attention: q/k per-head RMSNorm, NeoX RoPE at
// positions[b] (the (cos, sin) table [B][D/2] of the step) and the K/V
// append at row positions[b] done inside the attention kernel (raw fp32 q,
// k, v in), output bf16 [B][H][D]. D <= 256.
cudaError_t attention_launch_step(const float* q, const float* k, const float* v,
                                  const uint16_t* q_norm, const uint16_t* k_norm,
                                  const int32_t* tokens, int vocab, float eps, const float2* rope,
                                  uint16_t* kc, uint16_t* vc, const int32_t* positions, void* out,
                                  int B, int H, int Hkv, int D, int cap, float scale, void* ws,
                                  cudaStream_t st, bool pdl, const Prefetch* pf = nullptr,
                                  const OProjFuse* op = nullptr);
// Whether the step's attention can take o_proj into its cluster kernel
// (attention_launch_step with an OProjFuse) for this shape.
bool attention_oproj_fusable(int B, int H, int Hkv, int D, int cap, int hidden);
size_t attention_ws_bytes(int B, int H, int Hkv, int D, int cap);

// affine8 matmul on the tensor cores (gemm_affine8_sm100.cu): up to 3
// matrices sharing X bf16 [T][K], each Y [T][N] (+ residual); err is a
// device error word (nonzero after a device-side wait gave up).
struct A8Seg {
  const uint32_t* w;
  const uint16_t* s;
  const uint16_t* b;
  void* y;
  const float* res;
  int N;
  int y_bf16;
};
cudaError_t gemm_affine8_launch(const A8Seg* segs, int nseg, const uint16_t* X, int T, int K,
                                unsigned* err, cudaStream_t st, bool pdl, int* nt_used);
// The skinny variant (gemm_affine8_skinny.cu) for T <= 32 and K <= 2048,
// which gemm_affine8_launch takes by itself for those shapes.
bool gemm_affine8_skinny_ok(int T, int K);
cudaError_t gemm_affine8_skinny_launch(const A8Seg* segs, int nseg, const uint16_t* X, int T,
                                       int K, unsigned* err, cudaStream_t st, bool pdl);

// greedy token per row (argmax.cu); ws of argmax_ws_bytes(B, V) bytes
size_t argmax_ws_bytes(int B, int V);
cudaError_t argmax_launch(const float* logits, int B, int V, int32_t* out, void* ws,
                          cudaStream_t st, bool pdl);

}  // namespace qg
