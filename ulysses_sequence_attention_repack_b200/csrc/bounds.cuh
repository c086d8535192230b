// Range checks of computed global offsets, for the bounds-checked build.
//
// Built with -DULYSSES_DEBUG, every global access of the repack, prologue and
// push kernels (and the stores of the attention epilogue and of the backward)
// first checks that the span it touches lies inside the buffer the launch
// geometry describes.  An access outside is skipped and bit kErrBounds is set in the
// device error word, which ulysses_last_device_error reports; the kernel
// carries on (no trap, no assert), so the context stays usable.  In the
// default build the check is a compile-time `true` and costs nothing.
#pragma once

#include <cstdint>

namespace ulysses {

enum : uint32_t {
  kErrBounds = 4u,   // a computed global offset fell outside its buffer (checked build only)
};

#ifdef ULYSSES_DEBUG
constexpr bool kBoundsChecked = true;
#else
constexpr bool kBoundsChecked = false;
#endif

// True when elements [off, off + len) lie inside [0, extent).  kChecked
// selects the check independently of the build (the self-test uses it).
template <bool kChecked = kBoundsChecked>
__device__ __forceinline__ bool in_bounds(int64_t off, int64_t len, int64_t extent, unsigned int* err) {
  if (!kChecked) return true;
  if (off >= 0 && off + len <= extent) return true;
  if (err) atomicOr(err, kErrBounds);
  return false;
}

}  // namespace ulysses
