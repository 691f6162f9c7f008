// Softmax attention of many query rows at once (flash-attention style):
//
//   out[b][t][h] = sum_{s in keys(t)} softmax_s(q[b][t][h] . k[b][s][h/g] * scale) v[b][s][h/g]
//
// Definitions: fuel-transformers 0.19.1, src/models/lazy_quantized_whisper.rs,
// `multi_head_attn` (the Whisper encoder: every frame attends to every
// frame, scale 1/sqrt(d_head)); makima src/tts/qwen3/model.rs,
// `Qwen3Attention::forward` with `causal_mask` and `repeat_kv` (a prompt's
// rows attend causally to the cached rows before them and to themselves;
// query head h reads KV head h / (H/Hkv)). With `causal`, row t of T sits at
// position S - T + t and attends to keys [0, S - T + t]; otherwise to all S.
//
// Layout: bf16 rows addressed by strides (elements): element d of row t of
// head h of batch b at base + b*bs + t*ld + h*hs + d, for q, k, v (k and v
// share strides) and out. The Whisper layers use [T][H*D] rows; the prefill
// reads K/V straight from the decode cache [B][Hkv][cap][D].
//
// Kernel: one CTA of 4 warps per 64 query rows of one (head, batch); each
// warp owns 16 rows. Q stays in registers as mma fragments. Key blocks of 64
// rows of K and V are staged in shared memory by cp.async (two blocks in
// flight), 16-byte chunks XOR-swizzled by row so that ldmatrix reads are
// conflict-free. S = Q K^T and O += P V run on the tensor cores
// (mma.sync m16n8k16, bf16 operands, fp32 accumulation); the softmax is
// online in fp32 (exp2 with the scale folded in), per row over the quad of
// lanes that holds it. P is rounded to bf16 for the P V product and the
// same rounded values are summed for the denominator, so the rounding only
// reweights the rows (relative change of each weight at most 2^-8, bf16's
// unit roundoff).
#include "attention_rows.cuh"
#include "mma_sync.cuh"

namespace qg {
namespace ar {

constexpr int kWarps = 4;
constexpr int kRows = 16 * kWarps;  // query rows per CTA
constexpr int kKB = 64;             // key rows per block

using namespace mm;

template <int D>
__global__ void __launch_bounds__(kWarps * 32) attn_rows_kernel(const __grid_constant__ Params P) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* sQ = smem;                               // [kRows][D]
  uint8_t* sK = sQ + kRows * D * 2;                 // [2][kKB][D]
  uint8_t* sV = sK + 2 * kKB * D * 2;               // [2][kKB][D]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t4 = lane & 3;
  const int t0 = blockIdx.x * kRows, h = blockIdx.y, b = blockIdx.z;
  const int kvh = h / (P.H / P.Hkv);
  const uint16_t* qb = P.q + b * P.q_bs + h * P.q_hs;
  const uint16_t* kb = P.k + b * P.k_bs + kvh * P.k_hs;
  const uint16_t* vb = P.v + b * P.k_bs + kvh * P.k_hs;

  // keys this CTA needs: all S, or (causal) up to the last row's position
  const int off = P.S - P.T;  // position of query row 0
  int s_end = P.S;
  if (P.causal) s_end = min(P.S, off + min(P.T, t0 + kRows));
  const int nkb = (s_end + kKB - 1) / kKB;

  constexpr int CH = D / 8;  // 16-byte chunks per row
  // Q tile (rows past T zero-filled) and the first key block
  for (int i = tid; i < kRows * CH; i += kWarps * 32) {
    const int r = i / CH, c = i % CH;
    const bool ok = t0 + r < P.T;
    cp_async16(smem_u32(sQ) + swz<D>(r, c * 8), qb + (ok ? (long long)(t0 + r) * P.q_ld : 0) + c * 8, ok);
  }
  auto load_kv = [&](int blk, int buf) {
    const int s0 = blk * kKB;
    for (int i = tid; i < kKB * CH; i += kWarps * 32) {
      const int r = i / CH, c = i % CH;
      const bool ok = s0 + r < s_end;
      const long long ro = ok ? (long long)(s0 + r) * P.k_ld : 0;
      cp_async16(smem_u32(sK + buf * kKB * D * 2) + swz<D>(r, c * 8), kb + ro + c * 8, ok);
      cp_async16(smem_u32(sV + buf * kKB * D * 2) + swz<D>(r, c * 8), vb + ro + c * 8, ok);
    }
  };
  if (nkb > 0) load_kv(0, 0);
  cp_async_commit();

  // output accumulator: D/8 n-tiles of 16 x 8 per warp; running max and sum
  // of rows g and g + 8 of the warp's 16
  float oacc[D / 8][4];
#pragma unroll
  for (int j = 0; j < D / 8; ++j) oacc[j][0] = oacc[j][1] = oacc[j][2] = oacc[j][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  uint32_t qf[D / 16][4];
  const int row_a = t0 + warp * 16 + g, row_b = row_a + 8;  // this thread's two query rows
  const int pos_a = off + row_a, pos_b = off + row_b;

  for (int blk = 0; blk < nkb; ++blk) {
    const int buf = blk & 1;
    if (blk + 1 < nkb) load_kv(blk + 1, buf ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (blk == 0) {
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const int r = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int c = ks * 16 + (lane >> 4) * 8;
        ldsm_x4(smem_u32(sQ) + swz<D>(r, c), qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3]);
      }
    }
    const uint32_t kbase = smem_u32(sK + buf * kKB * D * 2);
    const uint32_t vbase = smem_u32(sV + buf * kKB * D * 2);
    // S = Q K^T for the block's 64 keys: 8 n-tiles of 8 keys
    float sc[kKB / 8][4];
#pragma unroll
    for (int j = 0; j < kKB / 8; ++j) sc[j][0] = sc[j][1] = sc[j][2] = sc[j][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
      for (int j = 0; j < kKB / 8; j += 2) {
        uint32_t b0, b1, b2, b3;
        const int r = j * 8 + (lane & 7) + (lane >> 4) * 8;
        const int c = ks * 16 + ((lane >> 3) & 1) * 8;
        ldsm_x4(kbase + swz<D>(r, c), b0, b1, b2, b3);
        mma_bf16(sc[j], qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], b0, b1);
        mma_bf16(sc[j + 1], qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], b2, b3);
      }
    }
    // scale, mask (keys past the end; causal), online softmax update
    const int s0 = blk * kKB;
    float mx0 = m0, mx1 = m1;
#pragma unroll
    for (int j = 0; j < kKB / 8; ++j) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int key = s0 + j * 8 + 2 * t4 + e;
        const bool in_a = key < s_end && (!P.causal || key <= pos_a);
        const bool in_b = key < s_end && (!P.causal || key <= pos_b);
        sc[j][e] = in_a ? sc[j][e] * P.scale_log2 : -INFINITY;
        sc[j][2 + e] = in_b ? sc[j][2 + e] * P.scale_log2 : -INFINITY;
        mx0 = fmaxf(mx0, sc[j][e]);
        mx1 = fmaxf(mx1, sc[j][2 + e]);
      }
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    // rows with no key yet keep max -inf: their weights are 0 (no NaN)
    const float a0 = mx0 == -INFINITY ? 1.f : exp2f(m0 - mx0);
    const float a1 = mx1 == -INFINITY ? 1.f : exp2f(m1 - mx1);
    const float base0 = mx0 == -INFINITY ? 0.f : mx0, base1 = mx1 == -INFINITY ? 0.f : mx1;
    l0 *= a0;
    l1 *= a1;
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
      oacc[j][0] *= a0;
      oacc[j][1] *= a0;
      oacc[j][2] *= a1;
      oacc[j][3] *= a1;
    }
    m0 = mx0;
    m1 = mx1;
    // O += P V: per 16 keys, P from two score tiles as the A fragment
#pragma unroll
    for (int kk = 0; kk < kKB / 16; ++kk) {
      float p[8];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        p[e] = bf16r(exp2f(sc[2 * kk][e] - base0));
        p[2 + e] = bf16r(exp2f(sc[2 * kk][2 + e] - base1));
        p[4 + e] = bf16r(exp2f(sc[2 * kk + 1][e] - base0));
        p[6 + e] = bf16r(exp2f(sc[2 * kk + 1][2 + e] - base1));
      }
      l0 += (p[0] + p[1]) + (p[4] + p[5]);
      l1 += (p[2] + p[3]) + (p[6] + p[7]);
      const uint32_t pa0 = pack_bf16(p[0], p[1]), pa1 = pack_bf16(p[2], p[3]);
      const uint32_t pa2 = pack_bf16(p[4], p[5]), pa3 = pack_bf16(p[6], p[7]);
#pragma unroll
      for (int j = 0; j < D / 8; j += 2) {
        uint32_t b0, b1, b2, b3;
        const int r = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int c = j * 8 + (lane >> 4) * 8;
        ldsm_x4_t(vbase + swz<D>(r, c), b0, b1, b2, b3);
        mma_bf16(oacc[j], pa0, pa1, pa2, pa3, b0, b1);
        mma_bf16(oacc[j + 1], pa0, pa1, pa2, pa3, b2, b3);
      }
    }
    __syncthreads();  // the buffer is refilled next iteration
  }
  cp_async_wait<0>();

  // finish: the row sums over the quad, normalise, store bf16
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const float i0 = l0 > 0.f ? 1.f / l0 : 0.f, i1 = l1 > 0.f ? 1.f / l1 : 0.f;
  uint16_t* ob = P.o + b * P.o_bs + h * P.o_hs;
#pragma unroll
  for (int j = 0; j < D / 8; ++j) {
    const int c = j * 8 + 2 * t4;
    if (row_a < P.T)
      *reinterpret_cast<uint32_t*>(ob + (long long)row_a * P.o_ld + c) =
          pack_bf16(oacc[j][0] * i0, oacc[j][1] * i0);
    if (row_b < P.T)
      *reinterpret_cast<uint32_t*>(ob + (long long)row_b * P.o_ld + c) =
          pack_bf16(oacc[j][2] * i1, oacc[j][3] * i1);
  }
}

template <int D>
constexpr int smem_bytes() {
  return (kRows + 4 * kKB) * D * 2;
}

}  // namespace ar

cudaError_t attn_rows_launch(const ar::Params& P, int B, int D, cudaStream_t st) {
  if (P.T == 0 || B == 0) return cudaSuccess;
  const dim3 grid((P.T + ar::kRows - 1) / ar::kRows, P.H, B);
  if (D == 64) {
    ensure_smem((const void*)ar::attn_rows_kernel<64>, ar::smem_bytes<64>());
    return launch_pdl(ar::attn_rows_kernel<64>, grid, dim3(ar::kWarps * 32),
                      (size_t)ar::smem_bytes<64>(), st, false, P);
  }
  ensure_smem((const void*)ar::attn_rows_kernel<128>, ar::smem_bytes<128>());
  return launch_pdl(ar::attn_rows_kernel<128>, grid, dim3(ar::kWarps * 32),
                    (size_t)ar::smem_bytes<128>(), st, false, P);
}

}  // namespace qg

using namespace qg;

extern "C" qg_status qg_attention_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                       uint16_t* out, int B, int T, int S, int H, int Hkv, int D,
                                       int causal, void* stream) {
  clear_error();
  QG_REQUIRE(B >= 0 && T >= 0 && S >= 0 && H >= 1 && Hkv >= 1, QG_ERR_UNSUPPORTED_SHAPE,
             "qg_attention_rows: B=%d T=%d S=%d H=%d Hkv=%d", B, T, S, H, Hkv);
  QG_REQUIRE(H % Hkv == 0, QG_ERR_UNSUPPORTED_SHAPE,
             "qg_attention_rows: H=%d must be a multiple of Hkv=%d", H, Hkv);
  QG_REQUIRE(D == 64 || D == 128, QG_ERR_UNSUPPORTED_SHAPE,
             "qg_attention_rows: D=%d must be 64 or 128", D);
  QG_REQUIRE(!causal || T <= S, QG_ERR_UNSUPPORTED_SHAPE,
             "qg_attention_rows: causal needs T=%d <= S=%d", T, S);
  QG_REQUIRE((long long)B * S * Hkv * D < (1LL << 40) && (long long)B * T * H * D < (1LL << 40),
             QG_ERR_UNSUPPORTED_SHAPE, "qg_attention_rows: too large");
  if (B == 0 || T == 0) return QG_OK;
  // with no keys (S = 0) k and v are never read and may be NULL
  QG_REQUIRE(q && out && (S == 0 || (k && v)), QG_ERR_INVALID_ARGUMENT,
             "qg_attention_rows: null pointer");
  QG_REQUIRE(aligned(q, 16) && aligned(k, 16) && aligned(v, 16) && aligned(out, 16),
             QG_ERR_MISALIGNED, "qg_attention_rows: q, k, v and out must be 16-byte aligned");
  ar::Params P = {};
  P.q = q;
  P.k = k;
  P.v = v;
  P.o = out;
  P.q_ld = (long long)H * D;
  P.q_hs = D;
  P.q_bs = (long long)T * H * D;
  P.k_ld = (long long)Hkv * D;
  P.k_hs = D;
  P.k_bs = (long long)S * Hkv * D;
  P.o_ld = P.q_ld;
  P.o_hs = D;
  P.o_bs = P.q_bs;
  P.T = T;
  P.S = S;
  P.H = H;
  P.Hkv = Hkv;
  P.causal = causal ? 1 : 0;
  P.scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
  attn_rows_launch(P, B, D, (cudaStream_t)stream);
  return check_launch("qg_attention_rows");
}
