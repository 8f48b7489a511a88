// pairs4096.cuh -- the pair step of the L = 8192 (M = 4096) on-chip kernels
// in "position layout".
//
// After the forward radix-16 stages, thread t holds positions 16 t + c
// (c < 16) of both chains; position 256 a + 16 b + c holds bin
// m = a + 16 b + 256 c.  The untangle / spectrum multiply / re-tangle of bin m
// needs the value at its partner bin: M - m (chain e, mod M) or M - 1 - m
// (chain o).  In position terms (t = 16 a + b):
//   chain o : partner of (t, c) is (255 - t, 15 - c)
//   chain e : t >= 16 -> (271 - t, 15 - c);  1 <= t <= 15 -> (16 - t, 15 - c);
//             t == 0 -> (0, (16 - c) mod 16); bins 0 and L share position 0,
//             bin M/2 (c = 8 of t = 0) is its own partner.
// Each thread evaluates the pair formula for its own 16 bins, reading the
// partner's value from a full-row copy of the partner's vector.  Both
// members of a pair compute the same formula from their own side, so no
// result has to be sent back.
//
// Spectrum row (per step and channel, 16L bytes), two planes:
//   plane 0: bf16 (re, im) pairs of K~ = (X + D) / 2L for all 2L bins of the
//            zero-padded transform X, entry spec8192_pos(f) holding bin f (the
//            order in which the tensor-core kernel reads it);
//   plane 1: complex64 (X + D) / 4L in position layout: entry
//            chain * 4096 + c * 256 + t holds the bin of position 16 t + c
//            (bin f = 2 m + chain); entry 0 packs the two real values
//            (K~[0], K~[L]) / 2.  The fp32 register kernel reads this plane.
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "fft_core.cuh"

namespace hyena {

// Entry of bin f = k1 + 16 k2 + 512 k3 in a plane of the L = 8192 spectrum
// row: the order in which the tensor-core kernel's spectrum pass reads it
// (thread (lane quarter Q, half h, lane) takes k1 = 4 Q + lane / 8,
// k2 = 4 (lane % 8) + T, k3 = 16 h + 4 i + e, one 16-byte load per (T, i)).
__host__ __device__ constexpr int spec8192_pos(int f) {
    return (((((f & 15) >> 2) * 2 + (f >> 13)) * 4 + ((f >> 4) & 3)) * 4 + ((f >> 11) & 3)) * 128 +
           (8 * (f & 3) + ((f >> 6) & 7)) * 4 + ((f >> 9) & 3);
}
constexpr int kSpec8192Plane = 16384;   // plane 0 entries (4 bytes each)

namespace p4096 {

constexpr int M = 4096;
constexpr int L = 8192;

// cos(pi s / 16), s = 0..8 and w_32^s = exp(-2 pi i s / 32), s = 0..15
__device__ __forceinline__ float cos16c(int s) {
    switch (s) {
        case 0: return 1.0f;
        case 1: return 0.98078528040323044913f;
        case 2: return 0.92387953251128675613f;
        case 3: return 0.83146961230254523708f;
        case 4: return 0.70710678118654752440f;
        case 5: return 0.55557023301960222474f;
        case 6: return 0.38268343236508977173f;
        case 7: return 0.19509032201612826785f;
        default: return 0.0f;
    }
}
__device__ __forceinline__ float2 w32c(int s) {
    const float c = s <= 8 ? cos16c(s) : -cos16c(16 - s);
    const float sn = cos16c(s <= 8 ? 8 - s : s - 8);
    return make_float2(c, -sn);
}

// Partner row of thread t's vector in chain e / chain o.
__device__ __forceinline__ int partner_row_e(int t) { return t >= 16 ? 271 - t : (16 - t) & 15; }
__device__ __forceinline__ int partner_row_o(int t) { return 255 - t; }

// Z at the own bin from the own value A, partner value B, own and partner
// spectrum values, and w = w_2L^f of the own bin f.
__device__ __forceinline__ float2 pair_own(float2 A, float2 B, float2 Kf, float2 Kg, float2 w) {
    const float2 S = cadd(A, cconj(B));
    const float2 T = cmul_i(cmul(w, csub(A, cconj(B))));
    const float2 Yf = cmul(csub(S, T), Kf);
    const float2 Yg = cmul(cconj(cadd(S, T)), Kg);
    const float2 P = cadd(Yf, cconj(Yg));
    const float2 U = cmul_i(cmulc(csub(Yf, cconj(Yg)), w));
    return cadd(P, U);
}

}  // namespace p4096
}  // namespace hyena
