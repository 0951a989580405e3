// bwd_gate.cuh -- which heads the backward takes from the tensor-core forward's saved values.
#pragma once

namespace efla {

// The saved values (every token's u and the state after every 64-token chunk, with the fp16
// operand rounding of the chunk products) are used only for heads whose keys have squared norm
// at most 16, whose a span at most a factor of 1024 and are all positive; the error of a
// reverse sweep fed by them grows with the keys' squared norm (emulated: dbeta's max error over
// its RMS 0.007 with ||k||^2 up to 16, 0.032 up to 100).  hs: per head {some a <= 0 (or NaN);
// max lambda; INT_MAX - min a; max a}, float bits as ints, gathered by the coefficient kernel.
__device__ __forceinline__ bool head_takes_saved(const int *hs, long long bh) {
    const int *h = hs + 4 * bh;
    const float lam_max = __int_as_float(h[1]), a_min = __int_as_float(0x7fffffff - h[2]);
    const float a_max = __int_as_float(h[3]);
    return h[0] == 0 && lam_max <= 16.f && a_max <= 1024.f * a_min;
}

}  // namespace efla
