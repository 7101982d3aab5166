// backward_mma.cuh -- the bf16 backward on the tensor cores (m16n8k16 bf16 MMA, fp32 accumulation).
//
// Same method as backward.cuh (FA-2's backward, scirs2-neural 0.4.3 flash_attention.rs
// flash_backward_head; GQA sums and RoPE undo from grouped_query_attention.rs): every product
// of the recurrence is a dense 16x8x16 MMA tile --
//   dq kernel   (4 warps x 16 query rows):   S = Q K^T, dP = dO V^T, dQ += dS K
//   dkdv kernel (4 warps x 16 keys):       S^T = K Q^T, dP^T = V dO^T, dV += P^T dO, dK += dS^T Q
// with the probabilities and dS formed in the accumulator registers and reused, rounded to
// bf16, as the A operand of the next product (no shared-memory round trip).  Tiles of 64 rows
// of Q, dO, K and V are staged in shared memory with a 16-byte XOR swizzle so that ldmatrix
// reads are conflict-free.  With RoPE the scores are recomputed from the rotated q and k carried
// as hi + lo bf16 pairs (S = Qh Kh^T + Qh Kl^T + Ql Kh^T, as in the forward), so P matches the
// forward's logsumexp; the gradient products use the hi halves.
#pragma once

#include "common.cuh"
#include "backward.cuh"

namespace attn {

constexpr int kBmThreads = 128;   // 4 warps x 16 rows = 64 rows per CTA
constexpr int kBmRows = 64;
constexpr int kBmTile = 64;       // keys (dq) / query rows (dkdv) per step
constexpr float kLog2e = 1.4426950408889634f;

// Byte offset of 16-byte chunk ch (8 bf16) of row r in a tile of rows of D bf16, with the low
// three chunk bits XOR-ed by the row: eight consecutive rows at one chunk hit eight banks groups.
template <int D>
__device__ __forceinline__ uint32_t bsw(int r, int ch) {
    return static_cast<uint32_t>(r * (D * 2) + (((ch & 7) ^ (r & 7)) | (ch & ~7)) * 16);
}

// Asynchronous copies global -> shared (cp.async, 16 or 4 bytes; a zero source size fills zeros).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, bool valid) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(valid ? 4 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Stage ROWS rows with cp.async: rows >= nvalid are zero-filled (their source address is row 0).
template <int D, int ROWS>
__device__ __forceinline__ void stage_rows_async(uint32_t tile, const __nv_bfloat16* src, long stride, int nvalid) {
    for (int idx = threadIdx.x; idx < ROWS * (D / 8); idx += kBmThreads) {
        const int r = idx / (D / 8), ch = idx % (D / 8);
        const bool ok = r < nvalid;
        cp_async16(tile + bsw<D>(r, ch), src + (ok ? r * stride : 0) + ch * 8, ok);
    }
}

struct BmParams {
    const __nv_bfloat16* q;     // [B, Sq, Hq, D]  (rotated hi half with RoPE)
    const __nv_bfloat16* ql;    // rotated lo half (RoPE only)
    const __nv_bfloat16* k;     // [B, Skv, Hkv, D] (rotated hi half with RoPE)
    const __nv_bfloat16* kl;    // rotated lo half (RoPE only)
    const __nv_bfloat16* v;
    const __nv_bfloat16* dout;  // [B, Sq, Hq, D]
    const float* lse;           // [B, Hq, Sq]
    const float* Dvec;          // [B, Hq, Sq]
    const float2* tab;          // (cos, sin) per [position][D/2] (RoPE only)
    float* g_f32;               // gradient output, fp32 or
    __nv_bfloat16* g_bf16;      // bf16
    float* g2_f32;              // dv (dkdv kernel)
    __nv_bfloat16* g2_bf16;
    int Hq, Hkv, Sq, Skv, q_pos0, causal;
    float scale;
    const float* mask;          // additive mask of the forward (MASK kernels), element strides:
    long mask_bs, mask_hs;      // batch, head; rows of Skv
};

// Store a 16-row x D accumulator fragment set (rows g, g+8 of the warp) with optional RoPE undo.
template <int D>
__device__ __forceinline__ void bm_store(float (&acc)[D / 8][4], float* f32, __nv_bfloat16* bf16, long row_off0,
                                         long row_off8, bool live0, bool live8, const float2* cs0, const float2* cs8,
                                         int t4) {
#pragma unroll
    for (int nd = 0; nd < D / 8; ++nd) {
        float x0 = acc[nd][0], x1 = acc[nd][1], y0 = acc[nd][2], y1 = acc[nd][3];
        const int pair = nd * 4 + t4;   // dims (8nd + 2t4, +1)
        if (cs0 != nullptr) rot_pair(x0, x1, cs0[pair], -1.f);
        if (cs8 != nullptr) rot_pair(y0, y1, cs8[pair], -1.f);
        const int d = nd * 8 + 2 * t4;
        if (f32 != nullptr) {
            if (live0) *reinterpret_cast<float2*>(f32 + row_off0 + d) = make_float2(x0, x1);
            if (live8) *reinterpret_cast<float2*>(f32 + row_off8 + d) = make_float2(y0, y1);
        } else {
            if (live0) *reinterpret_cast<uint32_t*>(bf16 + row_off0 + d) = pack_bf16x2(x0, x1);
            if (live8) *reinterpret_cast<uint32_t*>(bf16 + row_off8 + d) = pack_bf16x2(y0, y1);
        }
    }
}

// A fragments (16 rows x 16 dims, k step kk) of a swizzled tile, rows r0.. of the warp.
template <int D>
__device__ __forceinline__ void lda(uint32_t tile, int r0, int kk, int lane, uint32_t (&a)[4]) {
    const int m = lane >> 3;
    ldsm_x4(tile + bsw<D>(r0 + (m & 1) * 8 + (lane & 7), 2 * kk + (m >> 1)), a[0], a[1], a[2], a[3]);
}

// acc[nt] (16 x 8 for 8 rows nt of `tile`) += A(16 x D) * tile^T, over all k steps.  The two
// k steps that one ldmatrix brings in are issued in two passes over the eight accumulators, so
// consecutive MMAs never wait on each other's result.
template <int D, int NTB>
__device__ __forceinline__ void mma_rows_t(float (&acc)[NTB][4], uint32_t atile, int ar0, uint32_t btile, int lane) {
#pragma unroll
    for (int kk = 0; kk < D / 16; kk += 2) {
        uint32_t a0[4], a1[4], bh[NTB][2];
        lda<D>(atile, ar0, kk, lane, a0);
        lda<D>(atile, ar0, kk + 1, lane, a1);
#pragma unroll
        for (int nt = 0; nt < NTB; ++nt) {
            uint32_t b0, b1;
            ldsm_x4(btile + bsw<D>(nt * 8 + (lane & 7), 2 * kk + (lane >> 3)), b0, b1, bh[nt][0], bh[nt][1]);
            mma_bf16_16816(acc[nt], a0[0], a0[1], a0[2], a0[3], b0, b1);
        }
#pragma unroll
        for (int nt = 0; nt < NTB; ++nt) mma_bf16_16816(acc[nt], a1[0], a1[1], a1[2], a1[3], bh[nt][0], bh[nt][1]);
    }
}

// acc (16 x D) += A(16 x 16KS, given as bf16 fragments per 16-column step) * tile (16KS x D).
template <int D, int KS>
__device__ __forceinline__ void mma_p_tile(float (&acc)[D / 8][4], const uint32_t (&pa)[KS][4], uint32_t btile, int lane) {
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
        for (int nd = 0; nd < D / 8; nd += 2) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(btile + bsw<D>(ks * 16 + ((lane >> 3) & 1) * 8 + (lane & 7), nd + (lane >> 4)), b0, b1, b2, b3);
            mma_bf16_16816(acc[nd], pa[ks][0], pa[ks][1], pa[ks][2], pa[ks][3], b0, b1);
            mma_bf16_16816(acc[nd + 1], pa[ks][0], pa[ks][1], pa[ks][2], pa[ks][3], b2, b3);
        }
    }
}

// Round 16 x 8NTB fp32 accumulators (NTB column blocks of 8) to the bf16 A fragments of NTB/2
// k steps.
template <int NTB>
__device__ __forceinline__ void to_afrag(const float (&x)[NTB][4], uint32_t (&pa)[NTB / 2][4]) {
#pragma unroll
    for (int ks = 0; ks < NTB / 2; ++ks) {
        pa[ks][0] = pack_bf16x2(x[2 * ks][0], x[2 * ks][1]);
        pa[ks][1] = pack_bf16x2(x[2 * ks][2], x[2 * ks][3]);
        pa[ks][2] = pack_bf16x2(x[2 * ks + 1][0], x[2 * ks + 1][1]);
        pa[ks][3] = pack_bf16x2(x[2 * ks + 1][2], x[2 * ks + 1][3]);
    }
}

template <int D, bool ROPE>
struct BmCfg {
    // streamed rows per step (32 at D=128 removes the dk/dv kernel's register spills but costs
    // more in extra steps than it saves: 14.3 ms against 12.9 ms on a D=128, S=16384 backward)
    static constexpr int TT = kBmTile;
    static constexpr int NTB = TT / 8;                            // 8-column blocks of a score tile
    static constexpr int KS = TT / 16;                            // 16-row k steps of a P/dS product
    static constexpr int FIX = kBmRows * D * 2;                   // bytes of a 64-row bf16 tile
    static constexpr int STR = TT * D * 2;                        // bytes of a streamed tile
    static constexpr int NT = ROPE ? 3 : 2;                       // tiles per kind (K,Kl,V / Q,Ql,dO)
    static constexpr int STEP = NT * STR + 2 * TT * 4;            // + lse and D rows (dkdv)
    // fixed: Q, Ql, dO (dq) or K, Kl, V (dkdv); two buffers of the streamed step
    static constexpr int SMEM = NT * FIX + 2 * STEP + 128;
};

// dQ: CTA (64 query rows, q head h, batch b).
template <int D, bool ROPE, bool MASK>
__global__ void __launch_bounds__(kBmThreads, (D == 64 && !ROPE) ? 3 : 1) bwd_dq_mma_kernel(const BmParams p) {
    using C = BmCfg<D, ROPE>;
    extern __shared__ __align__(128) uint8_t bm_smem[];
    const uint32_t base = smem_u32(bm_smem);
    const uint32_t uQ = base, uQl = base + C::FIX, uG = base + (C::NT - 1) * C::FIX;
    auto uK = [&](int buf) { return base + C::NT * C::FIX + buf * C::STEP; };
    auto uKl = [&](int buf) { return uK(buf) + C::STR; };
    auto uV = [&](int buf) { return uK(buf) + (C::NT - 1) * C::STR; };
    const int h = blockIdx.y, b = blockIdx.z;
    const int kvh = h / (p.Hq / p.Hkv);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t4 = lane & 3;
    // causal: the last row blocks see the most keys, so they are scheduled first
    const int i0 = (p.causal ? static_cast<int>(gridDim.x) - 1 - static_cast<int>(blockIdx.x) : blockIdx.x) * kBmRows;
    const long qstride = static_cast<long>(p.Hq) * D, kstride = static_cast<long>(p.Hkv) * D;
    const long qbase = ((static_cast<long>(b) * p.Sq + i0) * p.Hq + h) * D;
    const int qvalid = min(kBmRows, p.Sq - i0);
    const long off_c = static_cast<long>(p.Skv) - p.Sq;
    const long last_row = static_cast<long>(i0) + kBmRows - 1;
    long kmax = p.causal ? last_row + off_c + 1 : p.Skv;
    kmax = kmax < 0 ? 0 : (kmax > p.Skv ? p.Skv : kmax);
    const int nsteps = static_cast<int>((kmax + C::TT - 1) / C::TT);
    auto issue_step = [&](int t) {
        const long k0 = static_cast<long>(t) * C::TT;
        const long kbase = ((static_cast<long>(b) * p.Skv + k0) * p.Hkv + kvh) * D;
        const int kvalid = static_cast<int>(min(static_cast<long>(C::TT), p.Skv - k0));
        stage_rows_async<D, C::TT>(uK(t & 1), p.k + kbase, kstride, kvalid);
        if (ROPE) stage_rows_async<D, C::TT>(uKl(t & 1), p.kl + kbase, kstride, kvalid);
        stage_rows_async<D, C::TT>(uV(t & 1), p.v + kbase, kstride, kvalid);
    };
    stage_rows_async<D, kBmRows>(uQ, p.q + qbase, qstride, qvalid);
    if (ROPE) stage_rows_async<D, kBmRows>(uQl, p.ql + qbase, qstride, qvalid);
    stage_rows_async<D, kBmRows>(uG, p.dout + qbase, qstride, qvalid);
    if (nsteps > 0) issue_step(0);
    cp_async_commit();
    // this thread's two rows: r_a = warp*16 + g, r_b = r_a + 8
    const int ra = i0 + warp * 16 + g, rb = ra + 8;
    auto row_state = [&](int i, float& lse2, float& dv, long& nvis) {
        if (i >= p.Sq) { lse2 = 0.f; dv = 0.f; nvis = 0; return; }
        const long srow = (static_cast<long>(b) * p.Hq + h) * p.Sq + i;
        const float l = p.lse[srow];
        lse2 = l * kLog2e;
        dv = p.Dvec[srow];
        long n = p.causal ? static_cast<long>(i) + off_c + 1 : p.Skv;
        n = n < 0 ? 0 : (n > p.Skv ? p.Skv : n);
        nvis = (l == -INFINITY) ? 0 : n;
    };
    float lse_a, lse_b, d_a, d_b;
    long nv_a, nv_b;
    row_state(ra, lse_a, d_a, nv_a);
    row_state(rb, lse_b, d_b, nv_b);
    float dq[D / 8][4];
#pragma unroll
    for (int nd = 0; nd < D / 8; ++nd)
#pragma unroll
        for (int e = 0; e < 4; ++e) dq[nd][e] = 0.f;
    const float sl2 = p.scale * kLog2e;
    for (int t = 0; t < nsteps; ++t) {
        // the next step's tiles load while this one is computed
        if (t + 1 < nsteps) issue_step(t + 1);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        const long k0 = static_cast<long>(t) * C::TT;
        const int buf = t & 1;
        float s[C::NTB][4], dp[C::NTB][4];
#pragma unroll
        for (int nt = 0; nt < C::NTB; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[nt][e] = dp[nt][e] = 0.f;
        mma_rows_t<D, C::NTB>(s, uQ, warp * 16, uK(buf), lane);
        if (ROPE) {
            mma_rows_t<D, C::NTB>(s, uQ, warp * 16, uKl(buf), lane);
            mma_rows_t<D, C::NTB>(s, uQl, warp * 16, uK(buf), lane);
        }
        mma_rows_t<D, C::NTB>(dp, uG, warp * 16, uV(buf), lane);
        // dS * scale in place of s
#pragma unroll
        for (int nt = 0; nt < C::NTB; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const long key = k0 + nt * 8 + 2 * t4 + (e & 1);
                const bool top = e < 2;
                const bool vis = key < (top ? nv_a : nv_b);
                float mb = 0.f;   // the forward's additive mask, in log2 units
                if (MASK && vis)
                    mb = __ldg(p.mask + b * p.mask_bs + h * p.mask_hs + static_cast<long>(top ? ra : rb) * p.Skv + key) *
                         kLog2e;
                const float pr = vis ? fast_exp2(s[nt][e] * sl2 + mb - (top ? lse_a : lse_b)) : 0.f;
                s[nt][e] = pr * (dp[nt][e] - (top ? d_a : d_b)) * p.scale;
            }
        }
        uint32_t pa[C::KS][4];
        to_afrag<C::NTB>(s, pa);
        mma_p_tile<D, C::KS>(dq, pa, uK(buf), lane);
        __syncthreads();   // buffer buf is refilled by the step after next
    }
    cp_async_wait<0>();
    const bool live_a = ra < p.Sq, live_b = rb < p.Sq;
    const long oa = ((static_cast<long>(b) * p.Sq + ra) * p.Hq + h) * D;
    const long ob = ((static_cast<long>(b) * p.Sq + rb) * p.Hq + h) * D;
    const float2* ca = (ROPE && live_a) ? p.tab + static_cast<long>(p.q_pos0 + ra) * (D / 2) : nullptr;
    const float2* cb = (ROPE && live_b) ? p.tab + static_cast<long>(p.q_pos0 + rb) * (D / 2) : nullptr;
    bm_store<D>(dq, p.g_f32, p.g_bf16, oa, ob, live_a, live_b, ca, cb, t4);
}

// dK, dV: CTA (64 keys, kv head, batch b); loops over the group's q heads and the query tiles.
template <int D, bool ROPE, bool MASK>
__global__ void __launch_bounds__(kBmThreads, (D == 64 && !ROPE) ? 3 : 1) bwd_dkdv_mma_kernel(const BmParams p) {
    using C = BmCfg<D, ROPE>;
    extern __shared__ __align__(128) uint8_t bm_smem[];
    const uint32_t base = smem_u32(bm_smem);
    const uint32_t uK = base, uKl = base + C::FIX, uV = base + (C::NT - 1) * C::FIX;
    auto uQ = [&](int buf) { return base + C::NT * C::FIX + buf * C::STEP; };
    auto uQl = [&](int buf) { return uQ(buf) + C::STR; };
    auto uG = [&](int buf) { return uQ(buf) + (C::NT - 1) * C::STR; };
    auto sLrow = [&](int buf) { return reinterpret_cast<float*>(bm_smem + C::NT * C::FIX + buf * C::STEP + C::NT * C::STR); };
    const int kvh = blockIdx.y, b = blockIdx.z;
    const int G = p.Hq / p.Hkv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t4 = lane & 3;
    const int j0 = blockIdx.x * kBmRows;
    const long qstride = static_cast<long>(p.Hq) * D, kstride = static_cast<long>(p.Hkv) * D;
    const long kbase = ((static_cast<long>(b) * p.Skv + j0) * p.Hkv + kvh) * D;
    const int kvalid = min(kBmRows, p.Skv - j0);
    const long off_c = static_cast<long>(p.Skv) - p.Sq;
    long i_lo = p.causal ? static_cast<long>(j0) - off_c : 0;
    i_lo = i_lo < 0 ? 0 : i_lo;
    const int t_start = static_cast<int>(i_lo / C::TT);
    const int t_per_head = (p.Sq + C::TT - 1) / C::TT - t_start;   // query tiles per q head
    const int nsteps = t_per_head > 0 ? t_per_head * G : 0;
    // step -> (group head, query tile); lse and D rows land after the step's tiles
    auto issue_step = [&](int t) {
        const int hg = t / t_per_head;
        const long i0 = static_cast<long>(t_start + t % t_per_head) * C::TT;
        const int h = kvh * G + hg;
        const long qbase = ((static_cast<long>(b) * p.Sq + i0) * p.Hq + h) * D;
        const int qvalid = static_cast<int>(min(static_cast<long>(C::TT), p.Sq - i0));
        stage_rows_async<D, C::TT>(uQ(t & 1), p.q + qbase, qstride, qvalid);
        if (ROPE) stage_rows_async<D, C::TT>(uQl(t & 1), p.ql + qbase, qstride, qvalid);
        stage_rows_async<D, C::TT>(uG(t & 1), p.dout + qbase, qstride, qvalid);
        const uint32_t dl = smem_u32(sLrow(t & 1));
        const long srow0 = (static_cast<long>(b) * p.Hq + h) * p.Sq + i0;
        for (int w = threadIdx.x; w < 2 * C::TT; w += kBmThreads) {
            const int r = w % C::TT;
            const bool ok = r < qvalid;
            const float* src = (w < C::TT ? p.lse : p.Dvec) + srow0 + (ok ? r : 0);
            cp_async4(dl + w * 4, src, ok);
        }
    };
    stage_rows_async<D, kBmRows>(uK, p.k + kbase, kstride, kvalid);
    if (ROPE) stage_rows_async<D, kBmRows>(uKl, p.kl + kbase, kstride, kvalid);
    stage_rows_async<D, kBmRows>(uV, p.v + kbase, kstride, kvalid);
    if (nsteps > 0) issue_step(0);
    cp_async_commit();
    const int ja = j0 + warp * 16 + g, jb = ja + 8;    // this thread's two keys
    float dk[D / 8][4], dv[D / 8][4];
#pragma unroll
    for (int nd = 0; nd < D / 8; ++nd)
#pragma unroll
        for (int e = 0; e < 4; ++e) dk[nd][e] = dv[nd][e] = 0.f;
    const float sl2 = p.scale * kLog2e;
    for (int t = 0; t < nsteps; ++t) {
        if (t + 1 < nsteps) issue_step(t + 1);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        const int buf = t & 1;
        const long i0 = static_cast<long>(t_start + t % t_per_head) * C::TT;
        const int qvalid = static_cast<int>(min(static_cast<long>(C::TT), p.Sq - i0));
        const float* sL = sLrow(buf);
        const float* sD = sL + C::TT;
        float s[C::NTB][4], dp[C::NTB][4];
#pragma unroll
        for (int nt = 0; nt < C::NTB; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[nt][e] = dp[nt][e] = 0.f;
        mma_rows_t<D, C::NTB>(s, uK, warp * 16, uQ(buf), lane);        // S^T = K Q^T
        if (ROPE) {
            mma_rows_t<D, C::NTB>(s, uK, warp * 16, uQl(buf), lane);
            mma_rows_t<D, C::NTB>(s, uKl, warp * 16, uQ(buf), lane);
        }
        mma_rows_t<D, C::NTB>(dp, uV, warp * 16, uG(buf), lane);       // dP^T = V dO^T
        // s <- P^T, dp <- dS^T * scale
#pragma unroll
        for (int nt = 0; nt < C::NTB; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int qi = nt * 8 + 2 * t4 + (e & 1);   // query row within the tile
                const long key = (e < 2) ? ja : jb;
                const float lse = sL[qi];
                const bool vis = qi < qvalid && key < p.Skv && lse != -INFINITY &&
                                 (!p.causal || key <= i0 + qi + off_c);
                float mb = 0.f;   // the forward's additive mask, in log2 units
                if (MASK && vis)
                    mb = __ldg(p.mask + b * p.mask_bs + static_cast<long>(kvh * G + (t / t_per_head)) * p.mask_hs +
                               (i0 + qi) * p.Skv + key) * kLog2e;
                const float pr = vis ? fast_exp2(s[nt][e] * sl2 + mb - lse * kLog2e) : 0.f;
                dp[nt][e] = pr * (dp[nt][e] - sD[qi]) * p.scale;
                s[nt][e] = pr;
            }
        }
        uint32_t pa[C::KS][4];
        to_afrag<C::NTB>(s, pa);
        mma_p_tile<D, C::KS>(dv, pa, uG(buf), lane);                   // dV += P^T dO
        to_afrag<C::NTB>(dp, pa);
        mma_p_tile<D, C::KS>(dk, pa, uQ(buf), lane);                   // dK += dS^T Q
        __syncthreads();   // buffer buf is refilled by the step after next
    }
    cp_async_wait<0>();
    const bool live_a = ja < p.Skv, live_b = jb < p.Skv;
    const long oa = ((static_cast<long>(b) * p.Skv + ja) * p.Hkv + kvh) * D;
    const long ob = ((static_cast<long>(b) * p.Skv + jb) * p.Hkv + kvh) * D;
    const float2* ca = (ROPE && live_a) ? p.tab + static_cast<long>(ja) * (D / 2) : nullptr;
    const float2* cb = (ROPE && live_b) ? p.tab + static_cast<long>(jb) * (D / 2) : nullptr;
    bm_store<D>(dk, p.g_f32, p.g_bf16, oa, ob, live_a, live_b, ca, cb, t4);
    bm_store<D>(dv, p.g2_f32, p.g2_bf16, oa, ob, live_a, live_b, nullptr, nullptr, t4);
}

// Rotated q/k for the MMA path: hi = bf16(x'), lo = bf16(x' - hi), x' the rotation in fp32.
__global__ void bwd_rope_split_kernel(const uint32_t* __restrict__ x, uint32_t* __restrict__ hi,
                                      uint32_t* __restrict__ lo, const float2* __restrict__ tab, long npairs,
                                      int S, int H, int D, int pos0) {
    const int half = D / 2;
    for (long idx = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; idx < npairs;
         idx += static_cast<long>(gridDim.x) * blockDim.x) {
        const int i = static_cast<int>(idx % half);
        const long row = idx / half;                 // (b*S + s)*H + h
        const int sidx = static_cast<int>((row / H) % S);
        const float2 r = tab[static_cast<long>(pos0 + sidx) * half + i];
        const uint32_t v = x[idx];
        float x0 = bf16lo_to_f32(v), x1 = bf16hi_to_f32(v);
        rot_pair(x0, x1, r, 1.f);
        const uint32_t h = pack_bf16x2(x0, x1);
        hi[idx] = h;
        lo[idx] = pack_bf16x2(x0 - bf16lo_to_f32(h), x1 - bf16hi_to_f32(h));
    }
}

// D_i = dO . O per row for the bf16 path: D/8 lanes per row, one 16-byte load of o and of dO per
// lane, the row's lanes reduced with shuffles.
template <int D>
__global__ void bwd_rowdot_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dout,
                                  float* __restrict__ Dvec, long nrows, int Sq, int Hq,
                                  const float* __restrict__ lse = nullptr, float* __restrict__ lse2 = nullptr) {
    constexpr int LPR = D / 8;                   // lanes per row (8 or 16)
    const long t = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
    const long row = t / LPR;
    const int part = static_cast<int>(t % LPR);
    float acc = 0.f;
    if (row < nrows) {
        const uint4 a = *reinterpret_cast<const uint4*>(o + row * D + part * 8);
        const uint4 c = *reinterpret_cast<const uint4*>(dout + row * D + part * 8);
        const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            acc = fmaf(bf16lo_to_f32(aw[e]), bf16lo_to_f32(cw[e]), acc);
            acc = fmaf(bf16hi_to_f32(aw[e]), bf16hi_to_f32(cw[e]), acc);
        }
    }
#pragma unroll
    for (int w = LPR / 2; w >= 1; w >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, w);
    if (row < nrows && part == 0) {
        const int h = static_cast<int>(row % Hq);
        const int i = static_cast<int>((row / Hq) % Sq);
        const long b = row / (static_cast<long>(Hq) * Sq);
        const long r = (b * Hq + h) * Sq + i;
        Dvec[r] = acc;
        // the tensor-core backward's log2-scaled LSE, same row order: rows with no visible key
        // (LSE = -inf) get +inf, so that exp2(s - L2) is 0 for them
        if (lse2 != nullptr) {
            const float l = lse[r];
            lse2[r] = l == -INFINITY ? INFINITY : l * 1.4426950408889634f;
        }
    }
}

}  // namespace attn
