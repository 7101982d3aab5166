// prefill_f32.cuh -- exact attention forward in float32 on the CUDA cores (FFMA, no TF32).
//
// Same semantics as the tensor-core bf16 kernel: tiles of 64 query rows x 64 keys, online
// softmax with a running row max m and row sum l (scirs2-neural 0.4.3 flash_attention.rs,
// online_softmax_update, with its "running max is -inf -> correction 0" guard), key tiles wholly
// above the causal diagonal skipped, output O / l and lse = m + ln l at the end.
//
// Thread layout: 256 threads = 64 rows x 4 threads; thread (r, c) holds dims [c*D/4, (c+1)*D/4)
// of query row r and of its output row.  Scores are reduced over the 4 threads with shuffles.
#pragma once

#include "common.cuh"

namespace attn {

template <int D>
__global__ void __launch_bounds__(256) prefill_f32_kernel(
    const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
    float* __restrict__ o, float* __restrict__ lse, int Hq, int Hkv, int Sq, int Skv, float scale,
    int causal, const float2* __restrict__ rope_tab, int q_pos0, const float* __restrict__ mask, long mask_bs,
    long mask_hs) {
    constexpr int BR = 64, BK = 64, DC = D / 4;
    extern __shared__ float smem_f32[];
    float* sK = smem_f32;            // [BK][D]
    float* sV = smem_f32 + BK * D;   // [BK][D]

    const int tid = threadIdx.x;
    const int r = tid >> 2, c = tid & 3;
    const int row0 = blockIdx.x * BR;
    const int h = blockIdx.y, b = blockIdx.z;
    const int kvh = h / (Hq / Hkv);
    const int i = row0 + r;                      // query row
    const long off = static_cast<long>(Skv) - Sq;
    const bool row_ok = i < Sq;

    float qr[DC], acc[DC];
#pragma unroll
    for (int d = 0; d < DC; ++d) {
        qr[d] = row_ok ? q[((static_cast<long>(b) * Sq + i) * Hq + h) * D + c * DC + d] : 0.f;
        acc[d] = 0.f;
    }
    if (rope_tab != nullptr && row_ok) {
        const float2* t = rope_tab + static_cast<long>(q_pos0 + i) * (D / 2) + c * (DC / 2);
#pragma unroll
        for (int p = 0; p < DC / 2; ++p) {
            const float x0 = qr[2 * p], x1 = qr[2 * p + 1];
            qr[2 * p] = x0 * t[p].x - x1 * t[p].y;
            qr[2 * p + 1] = x0 * t[p].y + x1 * t[p].x;
        }
    }

    float m = -INFINITY, l = 0.f;
    // last key any row of this block may see
    long kmax = causal ? (static_cast<long>(row0) + BR - 1 + off) : static_cast<long>(Skv) - 1;
    if (kmax > Skv - 1) kmax = Skv - 1;
    const int ntiles = kmax < 0 ? 0 : static_cast<int>(kmax / BK) + 1;
    const long my_last = causal ? static_cast<long>(i) + off : static_cast<long>(Skv) - 1;
    // additive mask row of this query (scirs2 / whisper-apr: score = dot * scale + mask[q, k])
    const float* mrow = (mask != nullptr && row_ok)
                            ? mask + b * mask_bs + h * mask_hs + static_cast<long>(i) * Skv : nullptr;

    for (int jt = 0; jt < ntiles; ++jt) {
        const int k0 = jt * BK;
        __syncthreads();
        for (int e = tid; e < BK * D; e += blockDim.x) {
            const int kk = e / D, d = e % D;
            const int j = k0 + kk;
            float kv = 0.f, vv = 0.f;
            if (j < Skv) {
                const long gi = ((static_cast<long>(b) * Skv + j) * Hkv + kvh) * D + d;
                kv = k[gi];
                vv = v[gi];
            }
            sK[e] = kv;
            sV[e] = vv;
        }
        __syncthreads();
        if (rope_tab != nullptr) {
            for (int e = tid; e < BK * (D / 2); e += blockDim.x) {
                const int kk = e / (D / 2), p = e % (D / 2);
                const int j = k0 + kk;
                if (j < Skv) {
                    const float2 t = rope_tab[static_cast<long>(j) * (D / 2) + p];
                    const float x0 = sK[kk * D + 2 * p], x1 = sK[kk * D + 2 * p + 1];
                    sK[kk * D + 2 * p] = x0 * t.x - x1 * t.y;
                    sK[kk * D + 2 * p + 1] = x0 * t.y + x1 * t.x;
                }
            }
            __syncthreads();
        }
        for (int kk = 0; kk < BK; ++kk) {
            const int j = k0 + kk;
            float part = 0.f;
#pragma unroll
            for (int d = 0; d < DC; ++d) part = fmaf(qr[d], sK[kk * D + c * DC + d], part);
            part += __shfl_xor_sync(0xffffffffu, part, 1);
            part += __shfl_xor_sync(0xffffffffu, part, 2);
            if (j >= Skv || static_cast<long>(j) > my_last) continue;   // masked key
            const float s = part * scale + (mrow != nullptr ? mrow[j] : 0.f);
            if (s == -INFINITY) continue;                               // masked by the additive mask
            const float mn = fmaxf(m, s);
            const float corr = (m == -INFINITY) ? 0.f : expf(m - mn);
            const float p = expf(s - mn);
            l = l * corr + p;
#pragma unroll
            for (int d = 0; d < DC; ++d) acc[d] = fmaf(p, sV[kk * D + c * DC + d], acc[d] * corr);
            m = mn;
        }
    }
    if (!row_ok) return;
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int d = 0; d < DC; ++d) o[((static_cast<long>(b) * Sq + i) * Hq + h) * D + c * DC + d] = acc[d] * inv;
    if (lse != nullptr && c == 0) lse[(static_cast<long>(b) * Hq + h) * Sq + i] = l > 0.f ? m + logf(l) : -INFINITY;
}

}  // namespace attn
