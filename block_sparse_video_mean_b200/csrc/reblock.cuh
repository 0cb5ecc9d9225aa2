// Spark-Reblock (whitened median bisection) — declared here, implemented below.
#pragma once
#include "spark_common.cuh"

namespace spark {

inline size_t reblock_workspace_bytes(int bh, int nb, int d) {
  (void)bh; (void)nb; (void)d;
  return 0;
}

inline int reblock_launch(int bh, int N, int nb, int d, const uint16_t* Q, const uint16_t* K,
                          const uint16_t* V, int32_t* perm, uint16_t* Qp, uint16_t* Kp,
                          uint16_t* Vp, int32_t* tree, void* ws, cudaStream_t stream) {
  (void)bh; (void)N; (void)nb; (void)d; (void)Q; (void)K; (void)V; (void)perm; (void)Qp;
  (void)Kp; (void)Vp; (void)tree; (void)ws; (void)stream;
  return SPARK_EUNSUPPORTED;
}

}  // namespace spark
