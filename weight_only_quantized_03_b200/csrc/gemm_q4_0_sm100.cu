// Q4_0 matmul on the tcgen05 tensor cores (sm_100a). Placeholder entry
// points until the kernel lands.
#include "qg_internal.cuh"

using namespace qg;

extern "C" size_t qg_gemm_q4_0_workspace_size(int M, int N, int K) {
  (void)M; (void)N; (void)K;
  return 0;
}

extern "C" qg_status qg_gemm_q4_0(const uint8_t* blocks, const float* A, const float* bias,
                                  float* C, int M, int N, int K, void* ws, size_t ws_bytes,
                                  void* stream) {
  clear_error();
  (void)blocks; (void)A; (void)bias; (void)C; (void)M; (void)N; (void)K; (void)ws;
  (void)ws_bytes; (void)stream;
  set_error("qg_gemm_q4_0: not available in this build");
  return QG_ERR_UNSUPPORTED_SHAPE;
}
