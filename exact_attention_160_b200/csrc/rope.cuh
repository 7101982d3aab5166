// rope.cuh -- rotary position embedding kernels.
//
// Rotation (scirs2-neural 0.4.4, grouped_query_attention.rs, RotaryPositionEmbedding::apply):
// pair p of a head vector at position pos turns by theta_p = pos * base^(-2p/D):
//   x'_2p   = x_2p cos(theta_p) - x_2p+1 sin(theta_p)
//   x'_2p+1 = x_2p sin(theta_p) + x_2p+1 cos(theta_p)
// Angles and their cosines/sines are formed in double precision (as the page does) and rounded
// to float32; the rotation itself runs in float32.
#pragma once

#include "common.cuh"

namespace attn {

__device__ __forceinline__ double rope_theta(double pos, int pair, int D, double base) {
    return pos / pow(base, 2.0 * static_cast<double>(pair) / static_cast<double>(D));
}

// tab[p * (D/2) + i] = (cos, sin) of theta_i at position p, for p in [0, P).
__global__ void rope_table_kernel(float2* __restrict__ tab, int P, int D, double base) {
    const int half = D / 2;
    const long n = static_cast<long>(P) * half;
    for (long idx = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; idx < n;
         idx += static_cast<long>(gridDim.x) * blockDim.x) {
        const int p = static_cast<int>(idx / half);
        const int i = static_cast<int>(idx % half);
        double s, c;
        sincos(rope_theta(static_cast<double>(p), i, D, base), &s, &c);
        tab[idx] = make_float2(static_cast<float>(c), static_cast<float>(s));
    }
}

// In-place rotation of x [T, H, D] at per-token positions pos[T].  One block per token: the
// block forms the token's D/2 angles once (double precision) and rotates every head with them.
template <typename T>
__global__ void rope_apply_kernel(T* __restrict__ x, const int32_t* __restrict__ pos, int ntok, int H,
                                  int D, double base) {
    extern __shared__ float2 cs[];   // [D/2]
    const int half = D / 2;
    for (int t = blockIdx.x; t < ntok; t += gridDim.x) {
        const double p = static_cast<double>(pos[t]);
        for (int i = threadIdx.x; i < half; i += blockDim.x) {
            double s, c;
            sincos(rope_theta(p, i, D, base), &s, &c);
            cs[i] = make_float2(static_cast<float>(c), static_cast<float>(s));
        }
        __syncthreads();
        T* xt = x + static_cast<long>(t) * H * D;
        for (int w = threadIdx.x; w < H * half; w += blockDim.x) {
            const int h = w / half, i = w % half;
            const float2 r = cs[i];
            if constexpr (sizeof(T) == 2) {
                uint32_t* pr = reinterpret_cast<uint32_t*>(xt + static_cast<long>(h) * D) + i;
                const uint32_t v = *pr;
                const float x0 = bf16lo_to_f32(v), x1 = bf16hi_to_f32(v);
                *pr = pack_bf16x2(x0 * r.x - x1 * r.y, x0 * r.y + x1 * r.x);
            } else {
                float2* pr = reinterpret_cast<float2*>(xt + static_cast<long>(h) * D) + i;
                const float2 v = *pr;
                *pr = make_float2(v.x * r.x - v.y * r.y, v.x * r.y + v.y * r.x);
            }
        }
        __syncthreads();
    }
}

// Rotated keys as an unevaluated bf16 pair: k' = hi + lo with hi = bf16(k'), lo = bf16(k' - hi),
// which keeps about 16 significant bits of the float32 rotation.  k, khi, klo: [B, S, Hkv, D]
// bf16; key j of every batch sits at position j; tab holds positions [0, S) or more.
__global__ void rope_split_kv_kernel(const uint32_t* __restrict__ k, uint32_t* __restrict__ khi,
                                     uint32_t* __restrict__ klo, const float2* __restrict__ tab,
                                     long npairs, int S, int Hkv, int D) {
    const int half = D / 2;
    for (long idx = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; idx < npairs;
         idx += static_cast<long>(gridDim.x) * blockDim.x) {
        const int i = static_cast<int>(idx % half);
        const long row = idx / half;                 // (b*S + j)*Hkv + kvh
        const int j = static_cast<int>((row / Hkv) % S);
        const float2 r = tab[static_cast<long>(j) * half + i];
        const uint32_t v = k[idx];
        const float x0 = bf16lo_to_f32(v), x1 = bf16hi_to_f32(v);
        const float y0 = x0 * r.x - x1 * r.y;
        const float y1 = x0 * r.y + x1 * r.x;
        const uint32_t hi = pack_bf16x2(y0, y1);
        khi[idx] = hi;
        klo[idx] = pack_bf16x2(y0 - bf16lo_to_f32(hi), y1 - bf16hi_to_f32(hi));
    }
}

}  // namespace attn
