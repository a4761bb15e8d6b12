// Workspace guards of the MOBA_DEBUG build: a 256-byte guard follows every
// carved region; each call fills the guards first and checks them last, so a
// kernel that wrote past the end of its region is reported (MOBA_ERR_CANARY,
// detail: the guard's number in carve order).  Release builds carve no guards
// and launch neither kernel.
#include "common.cuh"
#include "kernels.h"

namespace moba {
namespace {

__device__ __forceinline__ uint32_t guard_word(int g, int w) {
  return 0x5ca1ab1eu ^ ((uint32_t)g << 16) ^ (uint32_t)w;
}

__global__ void guard_fill_kernel(Guards gs) {
  for (int g = blockIdx.x; g < gs.n; g += gridDim.x)
    for (int w = threadIdx.x; w < kGuardWords; w += blockDim.x) gs.p[g][w] = guard_word(g, w);
}

__global__ void guard_check_kernel(Guards gs, DevPlan* plan) {
  for (int g = blockIdx.x; g < gs.n; g += gridDim.x)
    for (int w = threadIdx.x; w < kGuardWords; w += blockDim.x)
      if (gs.p[g][w] != guard_word(g, w)) raise_error(plan, kErrCanary, g);
}

}  // namespace

cudaError_t launch_guard_fill(const Guards& gs, cudaStream_t st) {
  if (gs.n <= 0) return cudaSuccess;
  guard_fill_kernel<<<gs.n, kGuardWords, 0, st>>>(gs);
  return cudaGetLastError();
}

cudaError_t launch_guard_check(const Guards& gs, DevPlan* plan, cudaStream_t st) {
  if (gs.n <= 0) return cudaSuccess;
  guard_check_kernel<<<gs.n, kGuardWords, 0, st>>>(gs, plan);
  return cudaGetLastError();
}

}  // namespace moba
