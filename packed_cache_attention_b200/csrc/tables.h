// Host-side constant tables of libkvq (see tables.cpp).
#pragma once
#include <cstdint>

namespace kvq {

// Width-w codebooks are packed back to back: centroids of width w start at 2^w - 2,
// thresholds of width w start at 2^w - w - 1.
constexpr int centroid_offset(int w) { return (1 << w) - 2; }
constexpr int threshold_offset(int w) { return (1 << w) - w - 1; }
constexpr int kCentroidCount = 510;   // sum of 2^w, w = 1..8
constexpr int kThresholdCount = 502;  // sum of 2^w - 1, w = 1..8

struct Tables {
  uint16_t centroid_f16[kCentroidCount];  // IEEE half bit patterns
  float threshold[kThresholdCount];
  float delta[9];                         // delta[0] = 1
  float nf4[16];
  float nf4_mid[15];
};

const Tables& tables();

}  // namespace kvq
