// checks.cuh -- range checks of the kernels' index arithmetic for the debug
// build (liblca_checked.so, compiled with -DLCA_CHECKS).
//
// LCA_CHECK(err, cond, where) guards one shared-memory, tensor-memory or
// global index: in the debug build a false `cond` sets the check bit of the
// device error word (and, if it is the first error, records `where`), and the
// guarded access is skipped; it never traps, so the context stays usable and
// the host reads LCA_ERR_DEVICE_CHECK from lca_get_device_error.  In the
// normal build every check is the constant `true` and costs nothing.
#pragma once

namespace lca {

constexpr int kErrCheck = 2;   // device error word bit: a range check failed

__device__ __forceinline__ bool check_failed(int* err, int where) {
  if (atomicOr(err, kErrCheck) == 0) atomicExch(err + 1, where);
  return false;
}

}  // namespace lca

#ifdef LCA_CHECKS
#define LCA_CHECK(err, cond, where) ((cond) ? true : ::lca::check_failed((err), (where)))
#else
#define LCA_CHECK(err, cond, where) true
#endif
