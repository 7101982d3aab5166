// backward_tc.cuh -- the bf16 backward on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// The method is FA-2's backward as scirs2-neural 0.4.3 (src/layers/flash_attention.rs,
// flash_backward_head) writes it, with the GQA group sum and the RoPE undo of scirs2-neural 0.4.4
// (grouped_query_attention.rs): from the forward's logsumexp L and D_i = dO_i . O_i,
//   P = exp(S - L),  dP = dO V^T,  dS = P o (dP - D),  dV = P^T dO,  dK = scale dS^T Q,  dQ = scale dS K.
// Two kernels, each with the forward's machinery (TMA tiles with 128-byte swizzle, an mbarrier
// ring, one MMA-issuing thread, fp32 accumulators in TMEM):
//   dq kernel   (CTA = 128 query rows of one q head):  S = Q K_j^T, dP = dO V_j^T (ss MMAs),
//               dQ += dS K_j (A = dS from TMEM) over the visible key tiles j.
//   dkdv kernel (CTA = 128 keys of one kv head):        S^T = K Q_i^T, dP^T = V dO_i^T (ss),
//               dV += P^T dO_i, dK += dS^T Q_i (A from TMEM) over every q head of the group and
//               every visible query tile i -- the group sum stays inside the CTA.
// The scores are recomputed rather than stored, so S and dP are formed in both kernels.
// P and dS are rounded to bf16 where they become MMA operands (written back over the first
// half of S / dP in TMEM).  With RoPE the scores come from the rotated q and k carried as hi + lo
// bf16 pairs (three product chains, as in the forward) and the gradient products use the hi
// halves; dq and dk are rotated back by the negated angle before they are stored.
//
// Warp roles: warp 0 TMA producer, warp 1 owns TMEM and issues the MMAs (one thread), warps 4-7
// and 8-11 are two compute warpgroups that share the 128 TMEM lanes of a tile (thread = one row:
// a query row in the dq kernel, a key in the dkdv kernel) and split its 128 columns in halves.
#pragma once

#include "backward.cuh"
#include "common.cuh"

namespace attn {

constexpr int kBtThreads = 384;
// Register split (setmaxnreg): the TMA/MMA warpgroup gives registers up, the two compute
// warpgroups (which hold S and dP rows, 128 values a thread) take them.  The launch must hold
// 128 * 72 + 256 * 216 registers (168 a thread); the host checks the compiled count.  Per
// sub-partition: (72 + 2 * 216) * 32 = 16128 <= 16384.
constexpr int kBtRegsControl = 72;
constexpr int kBtRegsCompute = 216;
constexpr int kBtLaunchRegsMin = (128 * kBtRegsControl + 256 * kBtRegsCompute + kBtThreads - 1) / kBtThreads;
// The dk/dv kernel forms P^T and dS^T elementwise (no reduction across a key's row), so its
// compute work splits into four warpgroups of 32 query columns each with no exchange: four warps
// per sub-partition hide each other's latencies.  640 threads launch with 96 registers each
// (five warps per sub-partition); setmaxnreg moves them to the compute warps: 56 x 128 +
// 104 x 512 = 60416 <= 96 x 640, and per sub-partition (56 + 4 * 104) * 32 = 15104 <= 16384.
constexpr int kBtKvWarpgroups = 4;
constexpr int kBtKvThreads = 128 + 128 * kBtKvWarpgroups;
constexpr int kBtKvRegsControl = 56;
constexpr int kBtKvRegsCompute = 104;
constexpr int kBtKvLaunchRegsMin =
    (128 * kBtKvRegsControl + 128 * kBtKvWarpgroups * kBtKvRegsCompute + kBtKvThreads - 1) / kBtKvThreads;

template <int D, bool ROPE>
struct BtCfg {
    static constexpr int TILE = 128 * D * 2;      // one 128-row bf16 tile
    static constexpr int NBOX = D / 64;           // 64-column TMA boxes per row
    static constexpr int BOX = TILE / NBOX;       // bytes of one box (16 KB)
    static constexpr int KSTEPS = D / 16;         // MMA K steps over the head dim
    static constexpr int NT = ROPE ? 3 : 2;       // tiles per set: (hi, lo,) other
    static constexpr int FIXED = NT * TILE;       // dq: Q (Ql) dO; dkdv: K (Kl) V
    static constexpr int ROWB = 1024;             // dkdv stage: the tile's log2 LSE and D rows (fp32)
    static constexpr int BUDGET = 232448 - 1024 - 512;
    static constexpr int STAGE_Q = NT * TILE;           // dq stage: K (Kl) V
    static constexpr int STAGE_K = NT * TILE + ROWB;    // dkdv stage: Q (Ql) dO, L2 row, D row
    static constexpr int STAGES_Q = (BUDGET - FIXED) / STAGE_Q > 4 ? 4 : (BUDGET - FIXED) / STAGE_Q;
    static constexpr int STAGES_K = (BUDGET - FIXED) / STAGE_K > 4 ? 4 : (BUDGET - FIXED) / STAGE_K;
    static constexpr int SMEM_Q = FIXED + STAGES_Q * STAGE_Q + 1024 + 512;
    static constexpr int SMEM_K = FIXED + STAGES_K * STAGE_K + 1024 + 512;
    static_assert(STAGES_Q >= 1 && STAGES_K >= 1, "stage budget");
    static_assert(SMEM_Q <= 232448 && SMEM_K <= 232448, "shared memory budget");
    // TMEM columns: [0,128) S or S^T (P / dS written over its first 64 columns), [128, 128+D) the
    // first accumulator (dQ or dV), [256,384) dP or dP^T (dS^T over its first 64 in dkdv),
    // [384, 384+D) dK.  Each ts product's A operand and accumulator share a half of TMEM.
    static constexpr uint32_t COL_S = 0, COL_ACC = 128, COL_DP = 256, COL_DK = 384;
    // dq kernel: S and dP in the first half; dQ and two dS buffers (dS(j) in buffer j % 2) in the
    // second, so S(j+1) and dP(j+1) can be computed while the compute warps still form dS(j).
    // (The dQ product's A operand, dS, and its accumulator share the second half.)
    static constexpr uint32_t DQ_COL_S = 0, DQ_COL_DP = 128, DQ_COL_ACC = 256, DQ_COL_DS = 384;
    // the pipelined order issues S(j+1) before dQ(j) releases stage j, so it needs two stages
    static constexpr bool DQ_PIPE = STAGES_Q >= 2;
    // dkdv kernel at D = 64: P^T and dS^T get buffers of their own (first half: S^T, dV, P^T;
    // second half: dP^T, dK, dS^T), so S^T(i+1) and dP^T(i+1) can be computed while the compute
    // warps still form P^T(i) and dS^T(i).  At D = 128 the accumulators leave no room.
    static constexpr bool KV_PIPE = D == 64 && STAGES_K >= 2;
    static constexpr uint32_t KV_COL_S = 0, KV_COL_DV = 128, KV_COL_PT = 192;
    static constexpr uint32_t KV_COL_DP = 256, KV_COL_DK = 384, KV_COL_DST = 448;
};

struct BtParams {
    const float* lse2;        // [B, Hq, Sq] log2-scaled LSE; +inf for rows that saw no key
    const float* Dvec;        // [B, Hq, Sq] D_i = dO_i . O_i
    const float2* tab;        // (cos, sin) per [position][D/2] (RoPE only)
    float* g_f32;             // dq (dq kernel) / dk (dkdv kernel): fp32, or
    __nv_bfloat16* g_bf16;    // bf16
    float* g2_f32;            // dv (dkdv kernel)
    __nv_bfloat16* g2_bf16;
    int B, Hq, Hkv, Sq, Skv, q_pos0, causal;
    float scale, scale_log2;
};

// Named barrier of the two compute warpgroups (256 threads): every thread has read its S / dP
// columns before any thread overwrites the first half of S / dP with bf16 operands.
template <int N = 256>
__device__ __forceinline__ void compute_sync() { asm volatile("bar.sync 1, %0;" ::"n"(N) : "memory"); }

// Store a row segment of n (= D/2) fp32 gradient values, optionally rotated back by -theta.
template <int N>
__device__ __forceinline__ void bt_store(const uint32_t (&acc)[N], float mul, const float2* cs, float* f32,
                                         __nv_bfloat16* bf16, long off) {
    float v[N];
#pragma unroll
    for (int e = 0; e < N; ++e) v[e] = __uint_as_float(acc[e]) * mul;
    if (cs != nullptr) {
#pragma unroll
        for (int e = 0; e < N; e += 2) rot_pair(v[e], v[e + 1], cs[e / 2], -1.f);
    }
    if (f32 != nullptr) {
        float4* dst = reinterpret_cast<float4*>(f32 + off);
#pragma unroll
        for (int e = 0; e < N / 4; ++e) dst[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
    } else {
        uint4* dst = reinterpret_cast<uint4*>(bf16 + off);
#pragma unroll
        for (int e = 0; e < N / 8; ++e)
            dst[e] = make_uint4(pack_bf16x2(v[8 * e], v[8 * e + 1]), pack_bf16x2(v[8 * e + 2], v[8 * e + 3]),
                                pack_bf16x2(v[8 * e + 4], v[8 * e + 5]), pack_bf16x2(v[8 * e + 6], v[8 * e + 7]));
    }
}

// Read N (16, 32 or 64) accumulator columns of this thread's TMEM lane.
template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[N]) {
    if constexpr (N == 16) {
        tmem_ld16(taddr, r);
    } else if constexpr (N == 32) {
        tmem_ld32(taddr, r);
    } else {
        uint32_t a[32], b[32];
        tmem_ld32(taddr, a);
        tmem_ld32(taddr + 32, b);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) r[e] = a[e], r[32 + e] = b[e];
    }
    tmem_wait_ld();
}

// Read D/2 accumulator columns [c0, c0 + D/2) of this thread's TMEM lane.
template <int D>
__device__ __forceinline__ void tmem_ld_half(uint32_t taddr, uint32_t (&r)[D / 2]) {
    if constexpr (D == 64) {
        tmem_ld32(taddr, r);
    } else {
        uint32_t a[32], b[32];
        tmem_ld32(taddr, a);
        tmem_ld32(taddr + 32, b);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) r[e] = a[e], r[32 + e] = b[e];
    }
    tmem_wait_ld();
}

// S-tile products issued from one thread: D[tmem] = sum over chains of A_c B_c^T (K-major tiles).
template <int D, bool ROPE>
__device__ __forceinline__ void bt_issue_scores(uint32_t d_tmem, uint32_t a_hi, uint32_t a_lo, uint32_t b_hi,
                                                uint32_t b_lo) {
    using C = BtCfg<D, ROPE>;
    constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false);
    constexpr uint32_t hiK = desc_sw128_hi(1024);
    constexpr int NCHAIN = ROPE ? 3 : 1;
#pragma unroll
    for (int ch = 0; ch < NCHAIN; ++ch) {
        const uint32_t a = desc_sw128_lo(ch == 2 ? a_lo : a_hi, 16);
        const uint32_t b = desc_sw128_lo(ch == 1 ? b_lo : b_hi, 16);
#pragma unroll
        for (int kk = 0; kk < C::KSTEPS; ++kk) {
            constexpr uint32_t box16 = C::BOX >> 4;
            const uint32_t off = (kk >> 2) * box16 + (kk & 3) * 2;
            mma_ss(d_tmem, desc_join(a + off, hiK), desc_join(b + off, hiK), idesc, (ch > 0 || kk > 0) ? 1u : 0u);
        }
    }
}

// acc[tmem] (+)= A[tmem, 128 x 128 bf16] * B, B a 128-row tile read MN-major (N = D).
template <int D, bool ROPE>
__device__ __forceinline__ void bt_issue_acc(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_tile, bool first) {
    using C = BtCfg<D, ROPE>;
    constexpr uint32_t idesc = idesc_bf16_f32(128, D, true);
    constexpr uint32_t hiK = desc_sw128_hi(1024);
    const uint32_t b = desc_sw128_lo(b_tile, C::BOX);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
        mma_ts(d_tmem, a_tmem + kk * 8, desc_join(b + kk * (2048 >> 4), hiK), idesc, (!first || kk > 0) ? 1u : 0u);
}

// ------------------------------------------------------------------------------------------
// dQ
// ------------------------------------------------------------------------------------------
template <int D, bool ROPE>
__global__ void __launch_bounds__(kBtThreads, 1) bwd_dq_tc_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_ql,
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_kl,
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do, const BtParams p) {
    using C = BtCfg<D, ROPE>;
    constexpr int ST = C::STAGES_Q;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;                                  // Q (hi), [Ql], dO
    uint8_t* sG = smem + (C::NT - 1) * C::TILE;
    uint8_t* sKV = smem + C::FIXED;                      // [ST][K (hi), [Kl], V]
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::FIXED + ST * C::STAGE_Q);
    uint64_t* bar_fix = bars + 0;
    uint64_t* bar_s_full = bars + 1;
    uint64_t* bar_p_ready = bars + 2;
    uint64_t* bar_acc_done = bars + 3;
    uint64_t* bar_final = bars + 4;
    uint64_t* bar_k_full = bars + 5;        // [ST]
    uint64_t* bar_v_full = bar_k_full + ST;
    uint64_t* bar_empty = bar_v_full + ST;
    uint64_t* bar_s_free = bar_empty + ST;  // the compute warps hold S(j), dP(j) in registers
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_s_free + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nqt = (p.Sq + 127) / 128;
    const int item = static_cast<int>(blockIdx.x);
    const int i = p.causal ? nqt - 1 - item / (p.B * p.Hq) : item / (p.B * p.Hq);   // heavy first
    const int rem = item % (p.B * p.Hq);
    const int b = rem / p.Hq, h = rem % p.Hq;
    const int kvh = h / (p.Hq / p.Hkv);
    const long off_c = static_cast<long>(p.Skv) - p.Sq;
    int nkv = (p.Skv + 127) / 128;
    if (p.causal) {
        const long last = static_cast<long>(i) * 128 + 127 + off_c;
        const long n = last < 0 ? 0 : last / 128 + 1;
        nkv = n < nkv ? static_cast<int>(n) : nkv;
    }

    if (tid == 0) {
        mbar_init(bar_fix, 1);
        mbar_init(bar_s_full, 1);
        mbar_init(bar_p_ready, 256);
        mbar_init(bar_acc_done, 1);
        mbar_init(bar_final, 1);
        for (int s = 0; s < ST; ++s) {
            mbar_init(bar_k_full + s, 1);
            mbar_init(bar_v_full + s, 1);
            mbar_init(bar_empty + s, 1);
        }
        mbar_init(bar_s_free, 256);
        mbar_fence_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    constexpr uint32_t cS = C::DQ_PIPE ? C::DQ_COL_S : C::COL_S;
    constexpr uint32_t cDP = C::DQ_PIPE ? C::DQ_COL_DP : C::COL_DP;
    constexpr uint32_t cACC = C::DQ_PIPE ? C::DQ_COL_ACC : C::COL_ACC;

    if (warp < 4) {
      setmaxnreg_dec<kBtRegsControl>();
      if (warp == 0) {
        if (lane == 0) {
            const uint64_t pol_q = l2_policy_evict_first();
            const uint64_t pol_kv = l2_policy_evict_last();
            mbar_arrive_expect_tx(bar_fix, C::FIXED);
            for (int bx = 0; bx < C::NBOX; ++bx) {
                tma_load_4d(&tm_q, bar_fix, sQ + bx * C::BOX, bx * 64, h, i * 128, b, pol_q);
                if (ROPE) tma_load_4d(&tm_ql, bar_fix, sQ + C::TILE + bx * C::BOX, bx * 64, h, i * 128, b, pol_q);
                tma_load_4d(&tm_do, bar_fix, sG + bx * C::BOX, bx * 64, h, i * 128, b, pol_q);
            }
            int issued = 0;
            for (int j = 0; j < nkv; ++j) {
                const int s = j % ST;
                if (!mbar_wait(bar_empty + s, ((j / ST) & 1) ^ 1)) break;
                issued = j + 1;
                uint8_t* st = sKV + s * C::STAGE_Q;
                mbar_arrive_expect_tx(bar_k_full + s, (C::NT - 1) * C::TILE);
                for (int bx = 0; bx < C::NBOX; ++bx) {
                    tma_load_4d(&tm_k, bar_k_full + s, st + bx * C::BOX, bx * 64, kvh, j * 128, b, pol_kv);
                    if (ROPE)
                        tma_load_4d(&tm_kl, bar_k_full + s, st + C::TILE + bx * C::BOX, bx * 64, kvh, j * 128, b, pol_kv);
                }
                uint8_t* sv = st + (C::NT - 1) * C::TILE;
                mbar_arrive_expect_tx(bar_v_full + s, C::TILE);
                for (int bx = 0; bx < C::NBOX; ++bx)
                    tma_load_4d(&tm_v, bar_v_full + s, sv + bx * C::BOX, bx * 64, kvh, j * 128, b, pol_kv);
            }
            // no copy may still be landing in shared memory when the CTA exits
            mbar_wait(bar_fix, 0);
            for (int j = issued - ST > 0 ? issued - ST : 0; j < issued; ++j) {
                mbar_wait(bar_k_full + j % ST, (j / ST) & 1);
                mbar_wait(bar_v_full + j % ST, (j / ST) & 1);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // per key tile j:  S(j) = Q K_j^T, dP(j) = dO V_j^T -> s_full; the compute warps
            // write dS(j) -> p_ready; dQ += dS(j) K_j; stage free.  Pipelined (two or more
            // stages): S(j+1), dP(j+1) are issued as soon as the compute warps have S(j), dP(j) in
            // registers (s_free), before dQ(j), so the tensor core computes them while dS(j) is
            // formed; dS(j) goes to its own buffer (j % 2), which dQ(j-2) -- issued before S(j),
            // hence complete by s_full(j) -- has finished reading.  Otherwise dS(j) is written
            // over S and S(j+1) follows dQ(j).
            bool ok = mbar_wait(bar_fix, 0);
            tc_fence_after();
            const uint32_t uQ = smem_u32(sQ), uG = smem_u32(sG);
            auto stage = [&](int j) { return smem_u32(sKV + (j % ST) * C::STAGE_Q); };
            auto issue_scores = [&](int j) {
                const uint32_t k = stage(j);
                bt_issue_scores<D, ROPE>(tmem + cS, uQ, uQ + C::TILE, k, k + C::TILE);
                bt_issue_scores<D, false>(tmem + cDP, uG, uG, k + (C::NT - 1) * C::TILE, 0);
                mma_commit(bar_s_full);
            };
            auto wait_kv = [&](int j) {
                const bool r = mbar_wait(bar_k_full + j % ST, (j / ST) & 1) && mbar_wait(bar_v_full + j % ST, (j / ST) & 1);
                tc_fence_after();
                return r;
            };
            if (ok && nkv > 0) {
                ok = wait_kv(0);
                if (ok) issue_scores(0);
            }
            for (int j = 0; j < nkv; ++j) {
                if (C::DQ_PIPE && j + 1 < nkv) {
                    if (ok) {
                        ok = mbar_wait(bar_s_free, j & 1);
                        tc_fence_after();
                    }
                    if (ok) ok = wait_kv(j + 1);
                    if (ok) issue_scores(j + 1);
                }
                if (ok) {
                    ok = mbar_wait(bar_p_ready, j & 1);
                    tc_fence_after();
                }
                const uint32_t aDS = C::DQ_PIPE ? tmem + C::DQ_COL_DS + 64 * (j & 1) : tmem + C::COL_S;
                if (ok) bt_issue_acc<D, ROPE>(tmem + cACC, aDS, stage(j), j == 0);
                mma_commit(bar_empty + j % ST);
                if (!C::DQ_PIPE && ok && j + 1 < nkv) {
                    ok = wait_kv(j + 1);
                    if (ok) issue_scores(j + 1);
                }
            }
            mma_commit(bar_acc_done);
            mma_commit(bar_final);
            mbar_wait(bar_final, 0);
        }
      }
    } else {
        setmaxnreg_inc<kBtRegsCompute>();
        const int wg = (warp - 4) >> 2;
        const int row = (warp & 3) * 32 + lane;
        const int qrow = i * 128 + row;
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_base + cS + 64 * wg;
        const uint32_t tP = tmem + lane_base + cDP + 64 * wg;
        const long lrow = (static_cast<long>(b) * p.Hq + h) * p.Sq + qrow;
        const bool live = qrow < p.Sq;
        const float l2 = live ? p.lse2[lrow] : INFINITY;
        const float dv = live ? p.Dvec[lrow] : 0.f;
        const long lim_causal = p.causal ? static_cast<long>(qrow) + off_c : static_cast<long>(p.Skv) - 1;
        const long lim = lim_causal < p.Skv - 1 ? lim_causal : static_cast<long>(p.Skv) - 1;
        const uint64_t sl2x2 = f2_pack(p.scale_log2, p.scale_log2);
        const uint64_t nl2x2 = f2_pack(-l2, -l2);
        const uint64_t ndvx2 = f2_pack(-dv, -dv);
        bool ok = true;
        for (int j = 0; j < nkv; ++j) {
            uint32_t sr[2][32], dr[2][32];
            if (ok && !__all_sync(0xffffffffu, mbar_wait(bar_s_full, j & 1))) ok = false;
            tc_fence_after();
            if (ok) {
                tmem_ld32(tS, sr[0]);
                tmem_ld32(tS + 32, sr[1]);
                tmem_ld32(tP, dr[0]);
                tmem_ld32(tP + 32, dr[1]);
                tmem_wait_ld();
            }
            const uint32_t tDS = C::DQ_PIPE ? tmem + lane_base + C::DQ_COL_DS + 64 * (j & 1) + 32 * wg
                                            : tmem + lane_base + C::COL_S + 32 * wg;
            if (C::DQ_PIPE) {
                // S(j), dP(j) are in registers: the MMA thread may overwrite them with S(j+1), dP(j+1)
                tc_fence_before();
                mbar_arrive(bar_s_free);
            } else {
                compute_sync();   // dS(j) is written over S(j), which the other warpgroup reads
            }
            if (ok) {
                const long k0 = static_cast<long>(j) * 128 + 64 * wg;   // first key of this half
                // keys past this row's causal limit or past Skv: S = -inf, so P = 0 and dS = 0.  A
                // separate pass, taken only by warps with such a key, keeps the loop below free of
                // per-element checks.
                if (__any_sync(0xffffffffu, k0 + 63 > lim)) {
#pragma unroll
                    for (int cb = 0; cb < 2; ++cb)
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (k0 + cb * 32 + e > lim) sr[cb][e] = __float_as_uint(-INFINITY);
                }
                uint32_t pk[2][16];
#pragma unroll
                for (int cb = 0; cb < 2; ++cb) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        float p0, p1;
                        f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[cb][2 * e]), __uint_as_float(sr[cb][2 * e + 1])),
                                         sl2x2, nl2x2),
                                  p0, p1);
                        p0 = fast_exp2(p0);
                        p1 = fast_exp2(p1);
                        const uint64_t t = f2_add(f2_pack(__uint_as_float(dr[cb][2 * e]), __uint_as_float(dr[cb][2 * e + 1])),
                                                  ndvx2);
                        float d0, d1;
                        f2_unpack(f2_mul(f2_pack(p0, p1), t), d0, d1);
                        pk[cb][e] = pack_bf16x2(d0, d1);
                    }
                }
                tmem_st16(tDS, pk[0]);
                tmem_st16(tDS + 16, pk[1]);
                tmem_wait_st();
            }
            tc_fence_before();
            mbar_arrive(bar_p_ready);
        }
        // epilogue: dQ = scale * acc, rotated back at the query's position with RoPE; the two
        // warpgroups store the two halves of the row
        bool have = ok && nkv > 0;
        if (have) {
            have = __all_sync(0xffffffffu, mbar_wait(bar_acc_done, 0));
            tc_fence_after();
        }
        uint32_t acc[D / 2];
        if (have) {
            tmem_ld_half<D>(tmem + lane_base + cACC + wg * (D / 2), acc);
        } else {
#pragma unroll
            for (int e = 0; e < D / 2; ++e) acc[e] = 0u;
        }
        if (live) {
            const long off = ((static_cast<long>(b) * p.Sq + qrow) * p.Hq + h) * D + wg * (D / 2);
            const float2* cs = ROPE ? p.tab + static_cast<long>(p.q_pos0 + qrow) * (D / 2) + wg * (D / 4) : nullptr;
            bt_store<D / 2>(acc, p.scale, cs, p.g_f32, p.g_bf16, off);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------------------------------
// dK, dV
// ------------------------------------------------------------------------------------------
template <int D, bool ROPE>
__global__ void __launch_bounds__(kBtKvThreads, 1) bwd_dkdv_tc_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_ql,
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_kl,
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
    const __grid_constant__ CUtensorMap tm_l2, const __grid_constant__ CUtensorMap tm_dv, const BtParams p) {
    using C = BtCfg<D, ROPE>;
    constexpr int ST = C::STAGES_K;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sK = smem;                                  // K (hi), [Kl], V
    uint8_t* sV = smem + (C::NT - 1) * C::TILE;
    uint8_t* sQS = smem + C::FIXED;                      // [ST][Q (hi), [Ql], dO, L2 row, D row]
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::FIXED + ST * C::STAGE_K);
    uint64_t* bar_fix = bars + 0;
    uint64_t* bar_s_full = bars + 1;
    uint64_t* bar_p_ready = bars + 2;
    uint64_t* bar_acc_done = bars + 3;
    uint64_t* bar_final = bars + 4;
    uint64_t* bar_full = bars + 5;          // [ST]
    uint64_t* bar_empty = bar_full + ST;
    uint64_t* bar_s_free = bar_empty + ST;  // KV_PIPE: the compute warps hold S^T(i), dP^T(i) in registers
    uint64_t* bar_pd_free = bar_s_free + 1; // KV_PIPE: dV(i), dK(i) completed (the P^T/dS^T buffers are free)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_pd_free + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nkt = (p.Skv + 127) / 128, nqt = (p.Sq + 127) / 128;
    const int G = p.Hq / p.Hkv;
    const int item = static_cast<int>(blockIdx.x);
    const int j = item / (p.B * p.Hkv);                  // causal: key tile 0 sees the most rows
    const int rem = item % (p.B * p.Hkv);
    const int b = rem / p.Hkv, kvh = rem % p.Hkv;
    const long off_c = static_cast<long>(p.Skv) - p.Sq;
    // query tiles that see a key of this tile: rows r with r + off >= 128 j
    int i0 = 0;
    if (p.causal) {
        const long r_first = static_cast<long>(j) * 128 - off_c;
        i0 = r_first <= 0 ? 0 : static_cast<int>(r_first / 128);
        if (i0 > nqt) i0 = nqt;
    }
    const int per_head = nqt - i0;
    const int n_it = G * per_head;
    (void)nkt;

    if (tid == 0) {
        mbar_init(bar_fix, 1);
        mbar_init(bar_s_full, 1);
        mbar_init(bar_p_ready, 128 * kBtKvWarpgroups);
        mbar_init(bar_acc_done, 1);
        mbar_init(bar_final, 1);
        for (int s = 0; s < ST; ++s) {
            mbar_init(bar_full + s, 1);
            mbar_init(bar_empty + s, 1);
        }
        mbar_init(bar_s_free, 128 * kBtKvWarpgroups);
        mbar_init(bar_pd_free, 1);
        mbar_fence_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    constexpr uint32_t cS = C::KV_PIPE ? C::KV_COL_S : C::COL_S;
    constexpr uint32_t cDP = C::KV_PIPE ? C::KV_COL_DP : C::COL_DP;
    constexpr uint32_t cDV = C::KV_PIPE ? C::KV_COL_DV : C::COL_ACC;
    constexpr uint32_t cDK = C::KV_PIPE ? C::KV_COL_DK : C::COL_DK;
    constexpr uint32_t cPT = C::KV_PIPE ? C::KV_COL_PT : C::COL_S;     // P^T (A of dV)
    constexpr uint32_t cDST = C::KV_PIPE ? C::KV_COL_DST : C::COL_DP;  // dS^T (A of dK)

    if (warp < 4) {
      setmaxnreg_dec<kBtKvRegsControl>();
      if (warp == 0) {
        if (lane == 0) {
            const uint64_t pol_kv = l2_policy_evict_first();
            const uint64_t pol_q = l2_policy_evict_last();
            mbar_arrive_expect_tx(bar_fix, C::FIXED);
            for (int bx = 0; bx < C::NBOX; ++bx) {
                tma_load_4d(&tm_k, bar_fix, sK + bx * C::BOX, bx * 64, kvh, j * 128, b, pol_kv);
                if (ROPE) tma_load_4d(&tm_kl, bar_fix, sK + C::TILE + bx * C::BOX, bx * 64, kvh, j * 128, b, pol_kv);
                tma_load_4d(&tm_v, bar_fix, sV + bx * C::BOX, bx * 64, kvh, j * 128, b, pol_kv);
            }
            int issued = 0;
            for (int it = 0; it < n_it; ++it) {
                const int s = it % ST;
                if (!mbar_wait(bar_empty + s, ((it / ST) & 1) ^ 1)) break;
                issued = it + 1;
                const int h = kvh * G + it / per_head, i = i0 + it % per_head;
                uint8_t* st = sQS + s * C::STAGE_K;
                mbar_arrive_expect_tx(bar_full + s, C::NT * C::TILE + C::ROWB);
                for (int bx = 0; bx < C::NBOX; ++bx) {
                    tma_load_4d(&tm_q, bar_full + s, st + bx * C::BOX, bx * 64, h, i * 128, b, pol_q);
                    if (ROPE) tma_load_4d(&tm_ql, bar_full + s, st + C::TILE + bx * C::BOX, bx * 64, h, i * 128, b, pol_q);
                    tma_load_4d(&tm_do, bar_full + s, st + (C::NT - 1) * C::TILE + bx * C::BOX, bx * 64, h, i * 128, b,
                                pol_q);
                }
                uint8_t* rows = st + C::NT * C::TILE;
                tma_load_2d(&tm_l2, bar_full + s, rows, i * 128, b * p.Hq + h, pol_q);
                tma_load_2d(&tm_dv, bar_full + s, rows + 512, i * 128, b * p.Hq + h, pol_q);
            }
            mbar_wait(bar_fix, 0);
            for (int it = issued - ST > 0 ? issued - ST : 0; it < issued; ++it) mbar_wait(bar_full + it % ST, (it / ST) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // per (q head, query tile) iteration:  S^T = K Q^T, dP^T = V dO^T -> s_full; the compute
            // warps write P^T and dS^T -> p_ready; dV += P^T dO, dK += dS^T Q; stage free.  KV_PIPE:
            // S^T(i+1), dP^T(i+1) are issued once the compute warps hold S^T(i), dP^T(i) in
            // registers (s_free), before dV(i), dK(i); P^T and dS^T have buffers of their own,
            // released by pd_free.  Otherwise P^T, dS^T are written over S^T, dP^T and the next
            // scores follow dV(i), dK(i).
            bool ok = mbar_wait(bar_fix, 0);
            tc_fence_after();
            const uint32_t uK = smem_u32(sK), uV = smem_u32(sV);
            auto stage = [&](int it) { return smem_u32(sQS + (it % ST) * C::STAGE_K); };
            auto issue_scores = [&](int it) {
                const uint32_t q = stage(it);
                bt_issue_scores<D, ROPE>(tmem + cS, uK, uK + C::TILE, q, q + C::TILE);
                bt_issue_scores<D, false>(tmem + cDP, uV, uV, q + (C::NT - 1) * C::TILE, 0);
                mma_commit(bar_s_full);
            };
            auto wait_q = [&](int it) {
                const bool r = mbar_wait(bar_full + it % ST, (it / ST) & 1);
                tc_fence_after();
                return r;
            };
            if (ok && n_it > 0) {
                ok = wait_q(0);
                if (ok) issue_scores(0);
            }
            for (int it = 0; it < n_it; ++it) {
                if (C::KV_PIPE && it + 1 < n_it) {
                    if (ok) {
                        ok = mbar_wait(bar_s_free, it & 1);
                        tc_fence_after();
                    }
                    if (ok) ok = wait_q(it + 1);
                    if (ok) issue_scores(it + 1);
                }
                if (ok) {
                    ok = mbar_wait(bar_p_ready, it & 1);
                    tc_fence_after();
                }
                if (ok) {
                    const uint32_t q = stage(it);
                    bt_issue_acc<D, ROPE>(tmem + cDV, tmem + cPT, q + (C::NT - 1) * C::TILE, it == 0);
                    bt_issue_acc<D, ROPE>(tmem + cDK, tmem + cDST, q, it == 0);
                }
                if (C::KV_PIPE) mma_commit(bar_pd_free);
                mma_commit(bar_empty + it % ST);
                if (!C::KV_PIPE && ok && it + 1 < n_it) {
                    ok = wait_q(it + 1);
                    if (ok) issue_scores(it + 1);
                }
            }
            mma_commit(bar_acc_done);
            mma_commit(bar_final);
            mbar_wait(bar_final, 0);
        }
      }
    } else {
        setmaxnreg_inc<kBtKvRegsCompute>();
        constexpr int CW = 128 / kBtKvWarpgroups;   // query columns of this warpgroup
        constexpr int AC = D / kBtKvWarpgroups;     // accumulator columns this warpgroup stores
        const int wg = (warp - 4) >> 2;
        const int row = (warp & 3) * 32 + lane;
        const int key = j * 128 + row;
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_base + cS + CW * wg;
        const uint32_t tP = tmem + lane_base + cDP + CW * wg;
        const uint32_t tPo = tmem + lane_base + cPT + (CW / 2) * wg;
        const uint32_t tDSo = tmem + lane_base + cDST + (CW / 2) * wg;
        const uint64_t sl2x2 = f2_pack(p.scale_log2, p.scale_log2);
        bool ok = true;
        for (int it = 0; it < n_it; ++it) {
            const int i = i0 + it % per_head;
            uint32_t sr[CW / 32][32], dr[CW / 32][32];
            if (ok && !__all_sync(0xffffffffu, mbar_wait(bar_s_full, it & 1))) ok = false;
            tc_fence_after();
            if (ok) {
#pragma unroll
                for (int cb = 0; cb < CW / 32; ++cb) {
                    tmem_ld32(tS + 32 * cb, sr[cb]);
                    tmem_ld32(tP + 32 * cb, dr[cb]);
                }
                tmem_wait_ld();
            }
            if (C::KV_PIPE) {
                // S^T(i), dP^T(i) are in registers: the MMA thread may overwrite them
                tc_fence_before();
                mbar_arrive(bar_s_free);
            } else {
                compute_sync<128 * kBtKvWarpgroups>();   // P^T, dS^T go over S^T, dP^T, which other warpgroups read
            }
            if (ok) {
                // this warpgroup's query columns q = 128 i + CW wg + c; the key is hidden from query
                // q past Sq, or (causal) when key > q + off
                const float* rows = reinterpret_cast<const float*>(sQS + (it % ST) * C::STAGE_K + C::NT * C::TILE);
                const float4* l2v = reinterpret_cast<const float4*>(rows + CW * wg);
                const float4* dvv = reinterpret_cast<const float4*>(rows + 128 + CW * wg);
                const long q0 = static_cast<long>(i) * 128 + CW * wg;
                // visible iff q < Sq and (not causal or q >= key - off)
                const long qmin = p.causal ? static_cast<long>(key) - off_c : 0;
                // hidden queries: S^T = -inf, so P^T = 0 and dS^T = 0 (a separate pass, taken only
                // by warps that have one, keeps the loop below free of per-element checks)
                if (__any_sync(0xffffffffu, q0 < qmin || q0 + CW - 1 >= p.Sq)) {
#pragma unroll
                    for (int cb = 0; cb < CW / 32; ++cb)
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const long qq = q0 + cb * 32 + e;
                            if (qq < qmin || qq >= p.Sq) sr[cb][e] = __float_as_uint(-INFINITY);
                        }
                }
                // 16 query columns at a time, stored as soon as they are formed (few live registers)
#pragma unroll
                for (int c = 0; c < CW / 16; ++c) {
                    uint32_t pp[8], pd[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int idx = c * 8 + e;                 // column pair 2 idx, 2 idx + 1
                        const int cb = idx >> 4, el = 2 * (idx & 15);
                        const float4 l4 = l2v[idx >> 1];
                        const float4 d4 = dvv[idx >> 1];
                        const float la = (idx & 1) ? l4.z : l4.x, lb = (idx & 1) ? l4.w : l4.y;
                        const float da = (idx & 1) ? d4.z : d4.x, db = (idx & 1) ? d4.w : d4.y;
                        float p0, p1;
                        f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[cb][el]), __uint_as_float(sr[cb][el + 1])), sl2x2,
                                         f2_pack(-la, -lb)),
                                  p0, p1);
                        p0 = fast_exp2(p0);
                        p1 = fast_exp2(p1);
                        const uint64_t t = f2_add(f2_pack(__uint_as_float(dr[cb][el]), __uint_as_float(dr[cb][el + 1])),
                                                  f2_pack(-da, -db));
                        float d0, d1;
                        f2_unpack(f2_mul(f2_pack(p0, p1), t), d0, d1);
                        pp[e] = pack_bf16x2(p0, p1);
                        pd[e] = pack_bf16x2(d0, d1);
                    }
                    if (C::KV_PIPE && c == 0 && it > 0) {
                        // the buffers still feed dV(i-1), dK(i-1) until those complete
                        if (!__all_sync(0xffffffffu, mbar_wait(bar_pd_free, (it - 1) & 1))) ok = false;
                        tc_fence_after();
                    }
                    tmem_st8(tPo + 8 * c, pp);
                    tmem_st8(tDSo + 8 * c, pd);
                }
                tmem_wait_st();
            }
            tc_fence_before();
            mbar_arrive(bar_p_ready);
        }
        // epilogue: dV = acc, dK = scale * acc rotated back at the key's position with RoPE; the
        // warpgroups store the two halves of the row
        bool have = ok && n_it > 0;
        if (have) {
            have = __all_sync(0xffffffffu, mbar_wait(bar_acc_done, 0));
            tc_fence_after();
        }
        uint32_t acc[AC];
        const bool live = key < p.Skv;
        const long off = ((static_cast<long>(b) * p.Skv + key) * p.Hkv + kvh) * D + wg * AC;
        if (have) {
            tmem_ld_cols<AC>(tmem + lane_base + cDV + wg * AC, acc);
        } else {
#pragma unroll
            for (int e = 0; e < AC; ++e) acc[e] = 0u;
        }
        if (live) bt_store<AC>(acc, 1.f, nullptr, p.g2_f32, p.g2_bf16, off);
        if (have) {
            tmem_ld_cols<AC>(tmem + lane_base + cDK + wg * AC, acc);
        }
        if (live) {
            const float2* cs = ROPE ? p.tab + static_cast<long>(key) * (D / 2) + wg * (AC / 2) : nullptr;
            bt_store<AC>(acc, p.scale, cs, p.g_f32, p.g_bf16, off);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}


}  // namespace attn
