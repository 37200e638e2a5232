// Launch accounting: a process-wide launch counter and an optional per-thread
// recorder that brackets every kernel launch with CUDA events on its stream and
// remembers the launch's algorithmic FLOPs and bytes. Used for live roofline
// measurement; recording works inside stream capture (the events become graph
// nodes) as long as the events were created by an earlier eager recording.
#pragma once

#include <cuda_runtime.h>

namespace sdp {

enum Family : int { F_GEMM = 0, F_ATTN = 1, F_GN_STATS = 2, F_GN_APPLY = 3, F_LN = 4, F_GEMV = 5, F_OTHER = 6 };

class Scope {
 public:
  // `kernels`: how many kernels the bracketed launch enqueues
  Scope(const char* kernel, int family, double flops, double bytes, cudaStream_t st, int kernels = 1);
  ~Scope();

 private:
  int slot_;
  unsigned int flags_;
  cudaStream_t st_;
};

}  // namespace sdp
