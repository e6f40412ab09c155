// Argument checks shared by the C-ABI entry points (host code only).
#pragma once

#include <cstddef>
#include <cstdint>

namespace ttt {
namespace abi {

inline bool misaligned(const void* p) {
  return p && (reinterpret_cast<uintptr_t>(p) & 15u) != 0;
}

// Do the byte ranges [a, a + na) and [b, b + nb) intersect? (null or empty: no)
inline bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + nb && b0 < a0 + na;
}

struct Span {
  const void* p;
  size_t n;
};

}  // namespace abi
}  // namespace ttt
