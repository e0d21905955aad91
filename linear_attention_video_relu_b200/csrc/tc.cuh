// tc.cuh -- tensor-core (tcgen05 + TMA) kernels for bf16 I/O.
#pragma once

#include "common.cuh"
#include "linattn.h"

namespace la {

struct TcArgs {
  int D;
  long long N;
  Rope rope;
  Sched sc;
  long long heads;
  const void *q, *k, *v, *g;
  void* out;
  int* flag;
  float2* gtab;
  float* part;
  float* apply;
  float* stS;
  float* stz;
  int use_state, commit, do_apply;
  float eps;
  cudaStream_t stream;
  void* const* events;
};

inline bool tc_supported(bool bf16, int D, int rope, int dt, int dh, int dw) {
  (void)bf16; (void)D; (void)rope; (void)dt; (void)dh; (void)dw;
  return false;
}
inline int tc_state_tile(int D) { return D == 128 ? 64 : 128; }
inline int tc_state_ctas_per_sm(int) { return 1; }
inline la_status tc_run(const TcArgs&) { return LA_ERR_UNSUPPORTED; }

}  // namespace la
