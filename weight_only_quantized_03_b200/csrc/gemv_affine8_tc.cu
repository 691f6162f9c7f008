// Affine-INT8 group-64 dequant GEMV on the tensor cores (the streaming
// path of qg_gemv_affine8_g64 for bf16 activations and B <= 32).
//
// Format and arithmetic as in gemv_affine8.cu (turbospark-runtime 0.3.0,
// src/qwen3_asr_metal.rs, PackedLinear / load_packed_linear; y = W x with
// w = q * s + beta per group of 64 columns).
//
// The packed codes go straight from HBM into the registers that form the
// mma operand: no shared-memory staging, no barriers on the hot path.
//
//   * mma.sync m16n8k16, fp16 operands, fp32 accumulation. A is 16 rows of
//     W: lane (g, t) loads 32 contiguous code bytes of row g and 32 of row
//     g + 8 with one 256-bit load each. A code byte q becomes the fp16 value
//     q - 128 with one byte permute and one packed subtract per two codes
//     (exact: fp16 has 11 significant bits). The k order inside an mma is free (a dot product
//     does not care), so k-slots {2t, 2t+1, 2t+8, 2t+9} of mma j are bytes
//     4j .. 4j+3 of lane t's 32-byte piece.
//   * B carries x with a group selector: column n = 2 b + h holds batch b's
//     x on the k-slots of 64-column group h of the 128-column chunk and zero
//     on the others. Lanes t = 0, 1 hold group 0 of a chunk and t = 2, 3
//     group 1, so one mma leaves both groups' partial sums
//     S_h = sum (q - 128) x apart, for 16 rows and 4 batch rows, already
//     reduced over the quad. Per group, y += s S + (beta + 128 s) sum(x):
//     the affine factorisation; no cross-lane reduction at all.
//   * x is converted once per CTA to fp16 in shared memory after a
//     power-of-two prescale 2^-e chosen from max|x| (so nothing overflows
//     fp16); bf16 values in fp16's normal range convert exactly, and the
//     outputs are multiplied back by 2^e. The prologue can also form x
//     itself from the previous op's fp32 outputs -- RMSNorm of the residual
//     stream or SiLU(gate) * up, rounded to bf16 exactly where the separate
//     kernels round -- so the decode step needs no launch for those ops.
//   * A warp streams 16-row blocks in 512-column super-chunks, four
//     128-column chunks of loads in flight per warp (64 registers). When
//     there are few blocks (small matrices), a team of S warps of one CTA
//     splits each block's columns and the partial sums meet in shared
//     memory in a fixed order (deterministic).
//   * Scales and biases of a super-chunk: lane (g, t) loads the bf16 pairs of
//     groups 2t, 2t + 1 for rows g and g + 8; chunk p takes them from lane
//     (g, p) by shuffle.
//   * A CTA holds up to 8 batch rows (two n-tiles). Past 8, the batch splits
//     into tiles of 8 along gridDim.y; the tiles stream the same weights at
//     about the same time, so HBM sees them about once and L2 serves the
//     rest (the CUDA-core path would be ALU-bound there).
#include <algorithm>

#include "gemv_tc.cuh"

namespace qg {
namespace gtc {

template <int NT, int W, bool BULK>
__global__ void __launch_bounds__(W * 32, 1)
    gemv_tc_kernel(const __grid_constant__ Params P) {
  extern __shared__ __align__(16) uint8_t smem[];
  tl_entry(P.tl);
  // the next kernel may be scheduled as soon as the weight loads are out (its
  // own wait still covers all of this one)
  gemv_tc_body<NT, W, BULK>(P, smem, [&] {
    pdl_trigger();
    pdl_wait();
    tl_wait(P.tl);
  });
  tl_exit(P.tl);
}

}  // namespace gtc


// Whether the tensor-core path takes this GEMV: bf16 x, 1 <= B <= 32, K a
// multiple of 512, codes 32-byte aligned (256-bit loads), scales and biases
// 4-byte aligned, and x fits in shared memory as fp16.
bool gemv_tc_eligible(const GemvSeg* segs, int nseg, int K, int B, bool x_f32) {
  if (x_f32 || K < gtc::kSC || K % gtc::kSC != 0 || B < 1 || B > gtc::kMaxBatch || nseg < 1 ||
      nseg > gtc::kMaxSegs)
    return false;
  for (int i = 0; i < nseg; ++i)
    if (!aligned(segs[i].w, 32) || !aligned(segs[i].s, 4) || !aligned(segs[i].b, 4)) return false;
  const int NT = B > 4 ? 2 : 1;
  return std::max(gtc_smem(K, NT, 16), gtc_smem(K, NT, 8)) <= 200 * 1024;
}

template <int NT, int W, bool BULK>
static cudaError_t gtc_launch_k(const gtc::Params& P, dim3 grid, cudaStream_t st, bool pdl) {
  const size_t smem = gtc_smem(P.K, NT, W);
  if (smem > 48 * 1024) ensure_smem((const void*)gtc::gemv_tc_kernel<NT, W, BULK>, 200 * 1024);
  return launch_pdl(gtc::gemv_tc_kernel<NT, W, BULK>, grid, dim3(W * 32), smem, st, pdl, P);
}
// the bulk instantiation for a bf16 x with more 128-column items per CTA
// (its first batch tile's rows times K / 128) than its warps keep in
// registers (three each)
template <int NT, int W>
static cudaError_t gtc_launch_nt(const gtc::Params& P, dim3 grid, cudaStream_t st, bool pdl) {
  const int bt = std::min(P.B, 4 * NT);
  const bool bulk = P.xmode == gtc::kXBf16 && bt * (P.K / 128) > 3 * W && aligned(P.x, 16);
  return bulk ? gtc_launch_k<NT, W, true>(P, grid, st, pdl)
              : gtc_launch_k<NT, W, false>(P, grid, st, pdl);
}

static cudaError_t gtc_launch(const GemvSeg* segs, int nseg, gtc::Params& P, int K, int B,
                              cudaStream_t st, bool pdl, const Prefetch* pf) {
  P.nseg = nseg;
  P.K = K;
  P.B = B;
  if (pf) P.pf = *pf;
  P.tl = tl_take(0);
  int blk = 0;
  for (int i = 0; i < nseg; ++i) {
    P.seg[i] = gtc::Seg{reinterpret_cast<const uint8_t*>(segs[i].w), segs[i].s, segs[i].b, segs[i].y,
                        segs[i].res, segs[i].N, segs[i].y_bf16, blk};
    blk += (segs[i].N + gtc::kRB - 1) / gtc::kRB;
  }
  P.nblocks = blk;
  if (blk == 0) return cudaSuccess;
  // One batch tile (B <= 4): 16 warps for matrices that stream (more
  // 16-row blocks than warp slots at 8 warps a CTA; 128 registers a thread),
  // 8 warps for the matrices of a decode layer, whose weights then all go
  // out before the wait. The 8-warp kernel takes the registers it needs
  // (about 234, no spills) at one CTA per SM: measured on the B200 in the
  // 0.6B step at batch 1, 813 us a step against 937 us when capped at 128
  // registers (two CTAs per SM, 136 bytes of spills a thread). Two batch
  // tiles: 8 warps (about 255 registers a thread). Batch tiles of
  // 8 rows along gridDim.y past B = 8: the tiles stream the same weights at
  // about the same time, so all but the first mostly hit L2.
  const int NT = B > 4 ? 2 : 1;
  const int sms = num_sms();
  const bool stream16 = NT == 1 && (long long)blk > 8LL * sms;
  const int W = stream16 ? 16 : 8;
  // batch tiles along gridDim.y share one wave of CTAs (one CTA per SM at
  // these register counts): each tile gets sms / tiles of them
  const int ny = (B + 4 * NT - 1) / (4 * NT);
  const int gx = std::max(1, std::min(blk, sms / ny));
  P.S = gtc_split(blk, K, W, gx);
  const dim3 grid(gx, ny);
  if (NT == 2) return gtc_launch_nt<2, 8>(P, grid, st, pdl);
  if (W == 16) return gtc_launch_nt<1, 16>(P, grid, st, pdl);
  return gtc_launch_nt<1, 8>(P, grid, st, pdl);
}

cudaError_t gemv_tc_launch(const GemvSeg* segs, int nseg, const void* x, int K, int B,
                           cudaStream_t st, bool pdl) {
  return gemv_tc_launch_pf(segs, nseg, x, K, B, st, pdl, nullptr);
}

cudaError_t gemv_tc_launch_pf(const GemvSeg* segs, int nseg, const void* x, int K, int B,
                              cudaStream_t st, bool pdl, const Prefetch* pf) {
  gtc::Params P = {};
  P.xmode = gtc::kXBf16;
  P.x = reinterpret_cast<const uint16_t*>(x);
  return gtc_launch(segs, nseg, P, K, B, st, pdl, pf);
}

cudaError_t gemv_tc_launch_rmsnorm(const GemvSeg* segs, int nseg, const float* x,
                                   const uint16_t* norm_w, float eps, int K, int B,
                                   cudaStream_t st, bool pdl, uint16_t* xout, const Prefetch* pf) {
  gtc::Params P = {};
  P.xmode = gtc::kXRmsNorm;
  P.xout = xout;
  P.xa = x;
  P.nw = norm_w;
  P.eps = eps;
  return gtc_launch(segs, nseg, P, K, B, st, pdl, pf);
}

cudaError_t gemv_tc_launch_rmsnorm_parts(const GemvSeg* segs, int nseg, const float* x,
                                         const float* parts, int nparts, float* xsum,
                                         const uint16_t* norm_w, float eps, int K, int B,
                                         cudaStream_t st, bool pdl, uint16_t* xout,
                                         const Prefetch* pf) {
  gtc::Params P = {};
  P.xmode = gtc::kXRmsNormParts;
  P.xout = xout;
  P.xa = x;
  P.parts = parts;
  P.nparts = nparts;
  P.xsum = xsum;
  P.nw = norm_w;
  P.eps = eps;
  return gtc_launch(segs, nseg, P, K, B, st, pdl, pf);
}

cudaError_t gemv_tc_launch_silu_mul(const GemvSeg* segs, int nseg, const float* gate,
                                    const float* up, int K, int B, cudaStream_t st, bool pdl,
                                    uint16_t* xout, const Prefetch* pf) {
  gtc::Params P = {};
  P.xmode = gtc::kXSiluMul;
  P.xout = xout;
  P.xa = gate;
  P.xb = up;
  return gtc_launch(segs, nseg, P, K, B, st, pdl, pf);
}

}  // namespace qg
