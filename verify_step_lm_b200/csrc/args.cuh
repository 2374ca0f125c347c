// Host-side argument checks shared by the extern "C" entry points (not part
// of the ABI): the limits include/mtpv.h states for the sampler calls.
#pragma once

#include <math.h>

namespace mtpv {

constexpr int kMaxK = 16;         // drafts per sequence
constexpr int kMaxV = 1 << 24;    // vocabulary
constexpr int kMaxRows = 65535;   // logits rows of one sampler launch (grid y)

inline bool verify_shape_ok(int B, int K, int V) {
    return B >= 1 && K >= 1 && K <= kMaxK && V >= 1 && V <= kMaxV &&
           (long long)B * (2 * K + 1) <= kMaxRows;
}

inline bool sampling_params_ok(float T, float top_p) {
    return isfinite(T) && T >= 0.0f && !isnan(top_p) && top_p > 0.0f;
}

}  // namespace mtpv
