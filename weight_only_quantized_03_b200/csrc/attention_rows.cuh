// Parameters of the multi-row attention kernel (attention_rows.cu), shared
// with its internal callers (the Whisper layer and the prefill).
#pragma once

#include "qg_internal.cuh"

namespace qg {
namespace ar {

// element d of row t of head h of batch b at base + b*bs + t*ld + h*hs + d
struct Params {
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  uint16_t* o;
  long long q_bs, q_ld, q_hs;
  long long k_bs, k_ld, k_hs;
  long long o_bs, o_ld, o_hs;
  int T, S, H, Hkv, causal;
  float scale_log2;  // scale * log2(e)
};

}  // namespace ar

cudaError_t attn_rows_launch(const ar::Params& P, int B, int D, cudaStream_t st);

}  // namespace qg
