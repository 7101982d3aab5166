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

constexpr int kRopeMaxHalf = 128;   // pairs whose denominators rope_table_kernel caches

__device__ __forceinline__ double rope_theta(double pos, int pair, int D, double base) {
    return pos / pow(base, 2.0 * static_cast<double>(pair) / static_cast<double>(D));
}

// tab[p * (D/2) + i] = (cos, sin) of theta_i at position p, for p in [0, P).  Dfreq is the head
// dim whose frequencies are used (the true dim when the vectors are zero-padded to D); pairs at
// or past Dfreq/2 are padding and get the identity (1, 0).
__global__ void rope_table_kernel(float2* __restrict__ tab, int P, int D, double base, int Dfreq) {
    // base^(2i/Dfreq) once per block (the same pow and division as rope_theta, so the table is
    // bit-identical to evaluating rope_theta per entry)
    __shared__ double denom[kRopeMaxHalf];
    const int half = D / 2;
    for (int i = threadIdx.x; i < half && i < kRopeMaxHalf; i += blockDim.x)
        denom[i] = pow(base, 2.0 * static_cast<double>(i) / static_cast<double>(Dfreq));
    __syncthreads();
    const long n = static_cast<long>(P) * half;
    for (long idx = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; idx < n;
         idx += static_cast<long>(gridDim.x) * blockDim.x) {
        const int p = static_cast<int>(idx / half);
        const int i = static_cast<int>(idx % half);
        if (2 * i >= Dfreq) {
            tab[idx] = make_float2(1.f, 0.f);
            continue;
        }
        double s, c;
        const double th = i < kRopeMaxHalf ? static_cast<double>(p) / denom[i] : rope_theta(static_cast<double>(p), i, Dfreq, base);
        sincos(th, &s, &c);
        tab[idx] = make_float2(static_cast<float>(c), static_cast<float>(s));
    }
}

// Zero-pad rows: dst rows of dst_words 32-bit words take the src_words of each src row followed
// by zeros (pads a head dim; src_words < dst_words).
__global__ void pad_rows_kernel(const uint32_t* __restrict__ src, uint32_t* __restrict__ dst, long rows,
                                int src_words, int dst_words) {
    const long n = rows * dst_words;
    for (long idx = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; idx < n;
         idx += static_cast<long>(gridDim.x) * blockDim.x) {
        const long r = idx / dst_words;
        const int c = static_cast<int>(idx % dst_words);
        dst[idx] = c < src_words ? src[r * src_words + c] : 0u;
    }
}

// Drop the padding: dst rows of dst_words words take the first dst_words of each src row.
__global__ void unpad_rows_kernel(const uint32_t* __restrict__ src, uint32_t* __restrict__ dst, long rows,
                                  int src_words, int dst_words) {
    const long n = rows * dst_words;
    for (long idx = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; idx < n;
         idx += static_cast<long>(gridDim.x) * blockDim.x) {
        const long r = idx / dst_words;
        const int c = static_cast<int>(idx % dst_words);
        dst[idx] = src[r * src_words + c];
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

// The same split with 16-byte accesses: thread = 8 consecutive elements (4 pairs) of one key
// row, with 32-bit index arithmetic.  Needs k, khi, klo and tab 16-byte aligned, D a multiple of
// 8 and rows * D / 8 < 2^31.
__global__ void rope_split_kv_vec_kernel(const uint4* __restrict__ k, uint4* __restrict__ khi, uint4* __restrict__ klo,
                                         const float4* __restrict__ tab, int nchunks, int S, int Hkv, int D) {
    const int cpr = D / 8;   // chunks per row
    for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < nchunks; idx += gridDim.x * blockDim.x) {
        const int row = idx / cpr, c = idx - row * cpr;   // row = (b*S + j)*Hkv + kvh
        const int j = (row / Hkv) % S;
        const float4* t = tab + (static_cast<long>(j) * (D / 2) + 4 * c) / 2;
        const float4 c01 = __ldg(t), c23 = __ldg(t + 1);
        const uint4 w = k[idx];
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
        const float cs[8] = {c01.x, c01.y, c01.z, c01.w, c23.x, c23.y, c23.z, c23.w};
        uint32_t hh[4], ll[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float x0 = bf16lo_to_f32(ww[e]), x1 = bf16hi_to_f32(ww[e]);
            const float cr = cs[2 * e], sr = cs[2 * e + 1];
            const float y0 = x0 * cr - x1 * sr;
            const float y1 = x0 * sr + x1 * cr;
            hh[e] = pack_bf16x2(y0, y1);
            ll[e] = pack_bf16x2(y0 - bf16lo_to_f32(hh[e]), y1 - bf16hi_to_f32(hh[e]));
        }
        khi[idx] = make_uint4(hh[0], hh[1], hh[2], hh[3]);
        klo[idx] = make_uint4(ll[0], ll[1], ll[2], ll[3]);
    }
}

// Decode-step cache update, fused (scirs2-neural 0.4.4 grouped_query_attention.rs,
// forward_with_cache: new keys/values go after the cached ones and new Q/K are rotated at the
// cache offset; whisper-apr 0.3.1 lfm2 KvCache: appending past the capacity is an error).
// One block per sequence b, so the block alone reads and advances seqlens[b]:
//   L = seqlens[b]; if L < 0 or L + T > Smax: set ATTN_DEVICE_ERR_OVERFLOW, leave b untouched.
//   for t < T: kcache[b, L+t] = rope(k_new[b, t], L+t); vcache[b, L+t] = v_new[b, t];
//              q[b, t] = rope(q[b, t], L+t) in place (q may be null);
//   seqlens[b] = L + T.
// All tensors bf16, rows of H*D contiguous elements; rope_base <= 0 copies without rotating.
__global__ void kv_append_kernel(uint32_t* __restrict__ kcache, uint4* __restrict__ vcache,
                                 int32_t* __restrict__ seqlens, const uint32_t* __restrict__ k_new,
                                 const uint4* __restrict__ v_new, uint32_t* __restrict__ q, int T, int Hq,
                                 int Hkv, int Smax, int D, double base) {
    extern __shared__ float2 cs[];   // [D/2] cos, sin of the current position
    __shared__ int s_len;
    const int b = blockIdx.x;
    const int half = D / 2;
    if (threadIdx.x == 0) {
        const int L = seqlens[b];
        const bool fits = L >= 0 && static_cast<long>(L) + T <= Smax;
        if (!fits) record_error(ATTN_DEVICE_ERR_OVERFLOW);
        s_len = fits ? L : -1;
    }
    __syncthreads();
    const int L = s_len;
    if (L < 0) return;
    const bool rot = base > 0.0;
    const int kpairs = Hkv * half;            // bf16 pairs in one key row
    const int vvec = Hkv * D / 8;             // 16-byte vectors in one value row
    const int qpairs = Hq * half;
    for (int t = 0; t < T; ++t) {
        const long pos = static_cast<long>(L) + t;
        if (rot) {
            for (int i = threadIdx.x; i < half; i += blockDim.x) {
                double sn, c;
                sincos(rope_theta(static_cast<double>(pos), i, D, base), &sn, &c);
                cs[i] = make_float2(static_cast<float>(c), static_cast<float>(sn));
            }
            __syncthreads();
        }
        const long src_row = static_cast<long>(b) * T + t;
        const long dst_row = static_cast<long>(b) * Smax + pos;
        for (int w = threadIdx.x; w < kpairs; w += blockDim.x) {
            uint32_t v = k_new[src_row * kpairs + w];
            if (rot) {
                const float2 r = cs[w % half];
                const float x0 = bf16lo_to_f32(v), x1 = bf16hi_to_f32(v);
                v = pack_bf16x2(x0 * r.x - x1 * r.y, x0 * r.y + x1 * r.x);
            }
            kcache[dst_row * kpairs + w] = v;
        }
        for (int w = threadIdx.x; w < vvec; w += blockDim.x) vcache[dst_row * vvec + w] = v_new[src_row * vvec + w];
        if (q != nullptr && rot) {
            for (int w = threadIdx.x; w < qpairs; w += blockDim.x) {
                uint32_t* pq = q + src_row * qpairs + w;
                const float2 r = cs[w % half];
                const uint32_t v = *pq;
                const float x0 = bf16lo_to_f32(v), x1 = bf16hi_to_f32(v);
                *pq = pack_bf16x2(x0 * r.x - x1 * r.y, x0 * r.y + x1 * r.x);
            }
        }
        __syncthreads();   // cs is rewritten for the next position
    }
    if (threadIdx.x == 0) seqlens[b] = L + T;
}

}  // namespace attn
