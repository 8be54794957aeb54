// Persistent decode kernel state (filled in by the decode-stack implementation).
#pragma once
#include "e0_device.cuh"

namespace e0 {

struct DecodeState {
  bool valid = false;
};

inline void decode_free(DecodeState &) {}

}  // namespace e0
