// Host-side helpers shared by the libpa translation units.
#pragma once

#include <cstdint>

namespace pa {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace pa
