// prefill_tc.cuh -- exact attention forward on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// The method (scirs2-neural 0.4.3, src/layers/flash_attention.rs): for a block of query rows,
// walk the key/value blocks; per block form S = Q K^T * scale, mask, and fold it into a running
// row max m and row sum l with the online-softmax recurrence (online_softmax_update):
//   m' = max(m, rowmax S);  l' = l e^(m-m') + sum e^(S-m');  O' = O e^(m-m') + e^(S-m') V
// skipping key blocks that lie wholly above the causal diagonal (flash_attention_forward), and
// finish with O / l and the logsumexp m + ln l.  Grouped-query head sharing follows
// scirs2-neural 0.4.4 grouped_query_attention.rs (q head h reads kv head h / (Hq/Hkv)).
//
// B200 design (not the pages' CPU loop structure):
//   * One CTA holds two 128-row query tiles that read the same K/V: two q heads of one GQA group
//     at the same rows when the group size is even, else two consecutive row tiles of one head.
//     Each K/V tile is therefore loaded once for 256 query rows.  A problem small enough that its
//     single tiles fit in one wave of the SMs runs one tile per CTA; at D=64 the CTA's two softmax
//     warpgroups then take alternate key tiles of that tile (interleaved keys, ILV), each with its
//     own online-softmax state, and the epilogue merges the two states (at D=128 the second
//     warpgroup idles).
//   * Warp roles (3 warpgroups): warp 0 issues TMA loads (Q once, then a ring of K/V stages);
//     warp 1 owns tensor memory; the tcgen05.mma of the CTA are issued from precomputed
//     shared-memory descriptors by one thread of warp 1 (D=128), or by one thread of warp 1 for
//     query tile 0 and one of warp 2 for tile 1 (D=64); warps 4-7 and 8-11 are the softmax
//     warpgroups of query tile 0 and 1, one thread per query row (a warp may only touch TMEM lanes
//     32*(warp%4) .. +31, so the row of a softmax thread is 32*(warp%4) + lane).
//   * S = Q K^T is a bf16 MMA (A and B from shared memory, M=128, N=128) into TMEM; the softmax
//     threads read their row of S with tcgen05.ld, compute P = exp2(S*scale*log2e - m) in fp32,
//     round P to bf16 and write it back to TMEM over S; O += P V is an MMA with A = P from TMEM
//     and B = V from shared memory (N = D), accumulating in TMEM.
//   * D=128: the MMA thread interleaves the tiles per KV tile j as PV_0(j), S_0(j+1), PV_1(j),
//     S_1(j+1): while one softmax warpgroup exponentiates its tile, the tensor core runs the other
//     tile's two products.  D=64 without RoPE: each tile's MMA thread issues PV_t(j) first half,
//     S_t(j+1), PV_t(j) second half (P's second half lives outside S's columns), so S_t(j+1) runs
//     while the second half of S_t(j) is exponentiated.  D=64 with RoPE (EARLY): P has columns of
//     its own, S_t(j+1) is issued as soon as the softmax holds S_t(j) in registers, and the two
//     softmax warpgroups take turns for their exponentials.
//   * Lazy rescale: the running max used for the exponent only moves when the block max exceeds
//     it by more than kRescaleThreshold (log2 units, 2^32), which keeps P <= 2^32 while skipping
//     the O correction (a tcgen05.ld/st of the row of O on the softmax's critical path) on all
//     but a few blocks even for peaked scores.  Nothing loses precision: P is rounded to bf16
//     relative to its own size, and l and O (fp32) stay far from overflow (l <= Skv 2^32).  The
//     "running max is -inf" guard makes rows with no visible key yet contribute nothing.
//   * With RoPE, Q is rotated in shared memory right after its TMA load and K arrives
//     pre-rotated; both carry hi + lo bf16 halves and S = Qh Kh^T + Qh Kl^T + Ql Kh^T.
//   * MASK instantiations add an additive score mask (whisper-apr attention_generated.rs,
//     compute_block_scores: score = dot * scale + mask) to the row of S in registers, as
//     mask / scale on the unscaled dot products, before the row max.  At D=64 without RoPE the
//     mask reaches shared memory by TMA (warps 2 and 3, swizzled boxes read conflict-free);
//     otherwise each thread loads its row from global memory.
//
// TMEM columns (512 allocated): tile t keeps S_t at [256t, 256t+128) and O_t after it (D columns,
// or 80 at D=64 with the ones block).  P_t (bf16 pairs, 64 columns) overwrites the first 64
// columns of S_t (D=128: S_t is fully in registers by then, and the next S_t MMA follows PV_t);
// at D=64 without RoPE its keys [64, 128) go to the 32 columns after O_t instead; with RoPE
// (EARLY) P_t has [256t+192, 256t+256) of its own.  TcCfg below has the exact offsets.
#pragma once

#include "common.cuh"

namespace attn {

constexpr int kTcThreads = 384;
// Register split between the warpgroups (setmaxnreg): the TMA/MMA warpgroup gives registers up,
// the two softmax warpgroups take them.  The launch must provide kTcThreads * kTcLaunchRegsMin
// registers, which covers 128 * kRegsControl + 256 * kRegsSoftmax; the host checks the compiled
// register count before every launch.  Per sub-partition (warps w, w+4, w+8 share one):
// (72 + 2 * 208) * 32 = 15616 <= 16384 registers.
constexpr int kRegsControl = 72;
constexpr int kRegsSoftmax = 208;
constexpr int kTcLaunchRegsMin = (128 * kRegsControl + 256 * kRegsSoftmax + kTcThreads - 1) / kTcThreads;
constexpr float kRescaleThreshold = 32.0f;
// RoPE forms of the kernel: none; K rotated beforehand into hi + lo halves (rope_split_kv_kernel);
// K loaded as it is and rotated into hi + lo halves in shared memory by the two idle warps of the
// control warpgroup (warps 2 and 3) while the ring runs ahead.
constexpr int kRopeNone = 0, kRopeKSplit = 1, kRopeKFused = 2;
// named barriers of the exponentiation turns (0 is __syncthreads), of the in-CTA merge and of
// one softmax warpgroup (4 + its index)
constexpr uint32_t kTcBarTurn0 = 1, kTcBarTurn1 = 2, kTcBarMerge = 3, kTcBarGroup0 = 4;
constexpr float kLn2 = 0.69314718055994531f;

template <int D, int ROPE, bool MASK = false>
struct TcCfg {
    static constexpr int BM = 128;                    // query rows per tile
    static constexpr int BN = 128;                    // keys per KV tile
    static constexpr int NBOX = D / 64;               // 128-byte-wide TMA boxes per row
    static constexpr int TILE_BYTES = BN * D * 2;     // one 128 x D bf16 tile
    static constexpr int KSTEPS = D / 16;             // MMA K steps of S = Q K^T
    // Masked D=64 without RoPE (MASK_TMA): the additive mask reaches shared memory by TMA in
    // 32-key x 128-row fp32 boxes (16 KB, 128-byte swizzle), MASK_SLOTS per query tile; the K/V
    // ring gives up a stage for them.
    static constexpr bool MASK_TMA = MASK && D == 64 && ROPE == 0;
    static constexpr int MASK_SLOTS = MASK_TMA ? 2 : 0;
    static constexpr int MASK_BOX_BYTES = 128 * 32 * 4;
    static constexpr int MASK_BYTES = 2 * MASK_SLOTS * MASK_BOX_BYTES;
    // D=128 with RoPE holds four Q tiles (hi, lo for both query tiles): one K/V stage fits.
    static constexpr int STAGES = (D == 64) ? (ROPE ? 3 : (MASK_TMA ? 3 : 4)) : (ROPE ? 1 : 2);
    static constexpr int K_TILES = ROPE ? 2 : 1;      // Kh, Kl
    static constexpr int Q_TILES = ROPE ? 2 : 1;      // Qh, Ql
    static constexpr int STAGE_BYTES = (K_TILES + 1) * TILE_BYTES;
    static constexpr int Q_BYTES = 2 * Q_TILES * TILE_BYTES;
    // D=64 with RoPE (EARLY): P_t has TMEM columns of its own, so S_t(j+1) -- three product
    // chains with RoPE -- is computed while the softmax still exponentiates S_t(j), and the two
    // softmax warpgroups take turns for their exponentials (each group's loads, row max, stores
    // and hand-offs run while the other one exponentiates).  Measured on B200: 8% faster for
    // GQA 32/8 RoPE B2 S4096; without RoPE (one chain) 2-7% slower than the layout below, so
    // only the RoPE kernels with pre-rotated K use it (the in-kernel K rotation needs warps 2
    // and 3, and warp 2 issues MMAs here).
    static constexpr bool EARLY = (D == 64 && ROPE == kRopeKSplit);
    // D=64 otherwise: the PV product runs with N = 80, its last 16 columns reading a block of
    // bf16 ones in shared memory, so column 64 of O accumulates the row sum of the rounded P the
    // MMA used (and every O correction rescales it with O).  One block serves every stage: the
    // descriptor of stage s reaches it through its leading-byte offset (ones - V_s).
    static constexpr bool ONES = (D == 64 && !EARLY);
    static constexpr int N_PV = ONES ? D + 16 : D;
    static constexpr int ONES_BYTES = ONES ? 128 * 128 : 0;
    static constexpr int SMEM_DATA = Q_BYTES + STAGES * STAGE_BYTES + ONES_BYTES + MASK_BYTES;
    static constexpr int SMEM_BYTES = SMEM_DATA + 1024 /* alignment slack */ + 512 /* barriers */;
    static_assert(8 * (16 + 5 * STAGES + 4 * MASK_SLOTS) + 4 <= 512, "barrier area");
    // TMEM columns: each query tile keeps S_t and O_t in one half of the 512 columns, S_t first;
    // P_t (bf16, 64 columns) is written over the first half of S_t once the softmax holds S_t in
    // registers.  (A P·V product whose A operand and accumulator lie in different halves ran
    // markedly slower on B200.)
    // EARLY: S_t, O_t (64) and P_t (64) fill the half: S0 [0,128) O0 [128,192) P0 [192,256),
    // S1 [256,384) O1 [384,448) P1 [448,512).
    // D=64 with the ones block (P_SPLIT): keys [0, 64) of P_t go over the first 32 columns of S_t,
    // keys [64, 128) into the 32 columns after O_t (O_t takes N_PV = 80 of the 128 after S_t), so
    // that S_t(j+1) may overwrite S_t as soon as the first half of PV_t(j) has read its P.
    static constexpr bool P_SPLIT = ONES;
    static constexpr uint32_t COL_S0 = 0, COL_O0 = 128, COL_P0 = EARLY ? 192 : 0;
    static constexpr uint32_t COL_S1 = 256, COL_O1 = 384, COL_P1 = EARLY ? 448 : 256;
    static constexpr uint32_t COL_PH0 = COL_O0 + N_PV, COL_PH1 = COL_O1 + N_PV;   // P_SPLIT: keys [64, 128)
    static_assert(!P_SPLIT || COL_PH1 + 32 <= 512, "TMEM columns");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct TcParams {
    __nv_bfloat16* o;         // bf16 output, or
    float* o_f32;             // fp32 output (when non-null)
    float* lse;
    const float2* rope_tab;   // [positions][D/2] (cos, sin), ROPE only
    int B, Hq, Hkv, Sq, Skv;
    int causal;
    int pair_heads;           // 1: tile pair = two heads of a group; 0: two row tiles of one head
    int single_tile;          // 1: one query tile per CTA (small problems: twice the CTAs)
    int q_pos0;
    int n_row_tiles;          // row tiles per head in the work decomposition
    int heads_per_item;       // Hq / 2 when pairing heads, Hq otherwise
    float scale_log2;         // scale * log2(e)
    const float* mask;        // additive mask on the scaled scores, or null
    long mask_bs, mask_hs;    // its batch and head strides (elements; 0 broadcasts); rows of Skv
    float inv_scale;          // 1 / scale: the mask enters the raw scores as mask / scale
    int mask_vec4;            // 1: every mask row starts 16-byte aligned (base, strides, Skv multiples of 4)
    int mask_tma;             // 1 (MASK_TMA kernels): the mask arrives by TMA through tm_m
    int kv_splits;            // >= 1; > 1 (single-tile mode only): each query tile's key tiles are
                              // divided among this many CTAs, which write partials
    float* o_part;            // [kv_splits][B][Sq][Hq][D] fp32 partial O, normalised per split
    float* lse_part;          // [kv_splits][B][Hq][Sq] partial logsumexp (natural log)
};

struct TcTile {
    int h;        // q head
    int r0;       // first query row
    int nkv;      // key tiles to process (0: nothing visible or inactive)
    bool active;
};

__device__ __forceinline__ int tc_kv_tiles(const TcParams& p, int r0) {
    const int nkv_all = (p.Skv + 127) / 128;
    if (!p.causal) return nkv_all;
    const long last = static_cast<long>(r0) + 127 + (static_cast<long>(p.Skv) - p.Sq);
    if (last < 0) return 0;
    const long n = last / 128 + 1;
    return n < nkv_all ? static_cast<int>(n) : nkv_all;
}

// ILV (interleaved keys, single-tile mode only): the two softmax warpgroups take alternate key
// tiles of the CTA's one query tile and the epilogue merges their states.  A template parameter,
// so that the other kernels carry none of its code.
template <int D, int ROPE, bool MASK, bool ILV>
__global__ void __launch_bounds__(kTcThreads, 1) prefill_tc_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_klo, const __grid_constant__ CUtensorMap tm_v,
    const __grid_constant__ CUtensorMap tm_o, const __grid_constant__ CUtensorMap tm_m, const TcParams p) {
    using C = TcCfg<D, ROPE, MASK>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;                                   // [2][Q_TILES][TILE_BYTES]
    uint8_t* sKV = smem + C::Q_BYTES;                     // [STAGES][(K_TILES+1)][TILE_BYTES]
    uint8_t* sOnes = sKV + C::STAGES * C::STAGE_BYTES;    // [128 keys][64] bf16 ones (ONES only)
    uint8_t* sMask = sOnes + C::ONES_BYTES;                // MASK_TMA: [2 tiles][MASK_SLOTS] 16 KB boxes
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::SMEM_DATA);
    uint64_t* bar_q_full = bars + 0;
    uint64_t* bar_q_ready = bars + 1;
    uint64_t* bar_s_full = bars + 2;       // [2] S_t(j) computed (commit after its MMAs)
    uint64_t* bar_p_ready = bars + 4;      // [2 tiles][2 halves] softmax t wrote keys [64h, 64h+64) of P_t(j)
    uint64_t* bar_o_done = bars + 8;       // [2] the last PV_t completed
    uint64_t* bar_mma_final = bars + 10;   // every MMA of the CTA completed
    uint64_t* bar_k_full = bars + 12;      // [STAGES]
    uint64_t* bar_v_full = bar_k_full + C::STAGES;
    uint64_t* bar_kv_empty = bar_v_full + C::STAGES;  // [STAGES], EARLY: [2 tiles][STAGES]
    uint64_t* bar_k_rot = bar_kv_empty + 2 * C::STAGES;   // [STAGES] K(j) rotated in place (kRopeKFused)
    uint64_t* bar_s_free = bar_k_rot + C::STAGES;     // [2] EARLY: softmax t holds S_t(j) in registers
    uint64_t* bar_pv_done = bar_s_free + 2;           // [2] EARLY: PV_t(j) completed (P_t free, O_t at rest)
    uint64_t* bar_m_full = bar_pv_done + 2;           // MASK_TMA: [2 tiles][MASK_SLOTS] mask box landed
    uint64_t* bar_m_empty = bar_m_full + 2 * C::MASK_SLOTS;   // [2 tiles][MASK_SLOTS] its softmax read it
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_m_empty + 2 * C::MASK_SLOTS);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;

    // ---- work item -> (batch, two query tiles) -------------------------------------------
    // consecutive CTAs are the key splits of one work item (kv_splits == 1: one CTA per item)
    const int split = static_cast<int>(blockIdx.x) % p.kv_splits;
    const int item = static_cast<int>(blockIdx.x) / p.kv_splits;
    const int items_per_rowtile = p.B * p.heads_per_item;
    const int rt = (p.n_row_tiles - 1) - item / items_per_rowtile;   // heavy first
    const int rem = item % items_per_rowtile;
    const int b = rem / p.heads_per_item;
    const int hi = rem % p.heads_per_item;
    // interleaved keys (below) need ring slots to spare: each step of the pair takes two
    static_assert(!ILV || C::STAGES >= 3, "interleaved keys need three K/V stages or more");
    constexpr bool ilv = ILV;
    // D=64 with the ones block (no RoPE): each query tile gets an MMA thread of its own (warps 1
    // and 2), as in the EARLY layout, so that neither tile's products wait behind the other
    // tile's hand-offs; a tcgen05.mma issue blocks while the tensor core is busy, which made one
    // thread issuing both tiles' products in a fixed order the pacing resource.
    // The masked kernel keeps one MMA thread and P over S: its softmax is bound by the per-row
    // mask loads, and the two groups' loads in step (which the per-tile MMA threads bring about)
    // measured 11% slower on B200.
    // (At D=128 an MMA thread per tile measured 1.27 ms on C5 against 0.97: there the tensor work
    // per step is twice as large and one thread's interleaved order keeps the pipe busier.)
    constexpr bool kOnesTwoIssuers = C::ONES && ROPE != kRopeKFused && !MASK;
    constexpr bool kPSplit = C::P_SPLIT && !MASK;   // P's second half after O (TMEM layout above)
    constexpr bool kPerTileMma = C::EARLY || kOnesTwoIssuers;   // one MMA thread per query tile
    TcTile tile[2];
    if (p.single_tile) {
        tile[0].h = tile[1].h = hi;
        tile[0].r0 = rt * 128;
        tile[1].r0 = ilv ? rt * 128 : p.Sq;    // the same rows, or inactive
    } else if (p.pair_heads) {
        tile[0].h = 2 * hi;
        tile[1].h = 2 * hi + 1;
        tile[0].r0 = tile[1].r0 = rt * 128;
    } else {
        tile[0].h = tile[1].h = hi;
        tile[0].r0 = rt * 256;
        tile[1].r0 = rt * 256 + 128;
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        tile[i].active = tile[i].r0 < p.Sq;
        tile[i].nkv = tile[i].active ? tc_kv_tiles(p, tile[i].r0) : 0;
    }
    // Key split (single-tile mode): this CTA takes a contiguous chunk of the tile's key tiles,
    // near-equal chunks with the remainder going to the first ones, and numbers them from 0 so
    // that every pipeline phase below runs as for a whole tile; only the key coordinates move.
    int kv0 = 0;
    if (p.kv_splits > 1) {
        const int n = tile[0].nkv, base = n / p.kv_splits, extra = n % p.kv_splits;
        kv0 = split * base + min(split, extra);
        tile[0].nkv = base + (split < extra ? 1 : 0);
    }
    // Interleaved keys: the CTA's key tiles u = 0, 1, 2, ... go alternately to the two softmax
    // warpgroups (tile t takes u = 2j + t at its step j), each running its own online softmax
    // over the same query rows.  Both then stream through the K/V ring in the order u, so every
    // ring slot serves one tile; without interleaving slot j serves both tiles' step j.
    const int n_keys = tile[0].nkv;   // this CTA's key tiles (interleaved mode)
    if (ilv) {
        tile[0].nkv = (n_keys + 1) / 2;
        tile[1].nkv = n_keys / 2;
    }
    const int kvh = tile[0].h / (p.Hq / p.Hkv);
    const int nkv = max(tile[0].nkv, tile[1].nkv);
    const int n_loads = ilv ? n_keys : nkv;   // K/V tiles through the ring
    // ring index (and key tile, from kv0) of tile t's step j
    auto ring_of = [ilv](int t, int j) { return ilv ? 2 * j + t : j; };

    // TMA copies, issued by thread 0: the query tiles, and K/V of ring index j into slot j % STAGES
    auto load_q = [&](uint64_t pol) {
        uint32_t qbytes = 0;
#pragma unroll
        for (int i = 0; i < 2; ++i)
            if (tile[i].active) qbytes += C::TILE_BYTES;
        mbar_arrive_expect_tx(bar_q_full, qbytes);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            if (!tile[i].active) continue;
            uint8_t* dst = sQ + i * C::Q_TILES * C::TILE_BYTES;
            for (int bx = 0; bx < C::NBOX; ++bx)
                tma_load_4d(&tm_q, bar_q_full, dst + bx * (C::TILE_BYTES / C::NBOX), bx * 64, tile[i].h, tile[i].r0, b,
                            pol);
        }
    };
    auto load_kv = [&](int j, uint64_t pol) {
        const int s = j % C::STAGES;
        uint8_t* st = sKV + s * C::STAGE_BYTES;
        // kRopeKFused: the raw K tile lands in the Kh slot and is rotated there
        mbar_arrive_expect_tx(bar_k_full + s, (ROPE == kRopeKSplit ? 2 : 1) * C::TILE_BYTES);
        for (int bx = 0; bx < C::NBOX; ++bx) {
            tma_load_4d(&tm_k, bar_k_full + s, st + bx * (C::TILE_BYTES / C::NBOX), bx * 64, kvh, (kv0 + j) * 128, b,
                        pol);
            if (ROPE == kRopeKSplit)
                tma_load_4d(&tm_klo, bar_k_full + s, st + C::TILE_BYTES + bx * (C::TILE_BYTES / C::NBOX), bx * 64, kvh,
                            (kv0 + j) * 128, b, pol);
        }
        uint8_t* sv = st + C::K_TILES * C::TILE_BYTES;
        mbar_arrive_expect_tx(bar_v_full + s, C::TILE_BYTES);
        for (int bx = 0; bx < C::NBOX; ++bx)
            tma_load_4d(&tm_v, bar_v_full + s, sv + bx * (C::TILE_BYTES / C::NBOX), bx * 64, kvh, (kv0 + j) * 128, b,
                        pol);
    };
    // the first ring loads find their slots free: issued during the set-up below
    const int n_pre = n_loads < C::STAGES ? n_loads : C::STAGES;

    // ---- set-up --------------------------------------------------------------------------
    if (tid == 0) {
        mbar_init(bar_q_full, 1);
        mbar_init(bar_q_ready, 256);   // both softmax warpgroups
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar_s_full + i, 1);
            mbar_init(bar_p_ready + 2 * i, 128);
            mbar_init(bar_p_ready + 2 * i + 1, 128);
            mbar_init(bar_o_done + i, 1);
        }
        mbar_init(bar_mma_final, kPerTileMma ? 2 : 1);   // one commit per MMA thread
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(bar_k_full + s, 1);
            mbar_init(bar_v_full + s, 1);
            mbar_init(bar_kv_empty + s, 1);                  // one commit from the (tile 0) MMA thread
            mbar_init(bar_kv_empty + C::STAGES + s, 1);      // EARLY: one from the tile-1 MMA thread
            mbar_init(bar_k_rot + s, C::EARLY ? 32 : 64);    // the rotating warps' threads
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar_s_free + i, 128);
            mbar_init(bar_pv_done + i, 1);
        }
        for (int i = 0; i < 2 * C::MASK_SLOTS; ++i) {
            mbar_init(bar_m_full + i, 1);
            mbar_init(bar_m_empty + i, 128);   // every thread of the tile's softmax warpgroup
        }
        mbar_fence_init();
        // The copies go out now, while the tensor memory is allocated and the block synchronises
        // (the barriers they signal are initialised; nothing else touches their destinations).
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        if (ROPE == kRopeKSplit) tma_prefetch_desc(&tm_klo);
        load_q(l2_policy_evict_first());
        const uint64_t pol_kv = l2_policy_evict_last();
        for (int j = 0; j < n_pre; ++j) load_kv(j, pol_kv);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    if (C::ONES) {
        // bf16 1.0 everywhere (the swizzle only permutes it), visible to the tensor core
        uint4* o4 = reinterpret_cast<uint4*>(sOnes);
        for (int i = tid; i < C::ONES_BYTES / 16; i += kTcThreads) o4[i] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp < 4) {
      setmaxnreg_dec<kRegsControl>();
      if (warp == 0) {
        // =============================== TMA producer ===================================
        if (lane == 0) {
            const uint64_t pol_kv = l2_policy_evict_last();
            int issued = n_pre;   // the query tiles and ring loads [0, n_pre) went out in the set-up
            for (int j = n_pre; j < n_loads; ++j) {
                const int s = j % C::STAGES;
                const uint32_t ph = (j / C::STAGES) & 1;
                // EARLY: each MMA thread releases the stages its own tile used (j - STAGES < n_t);
                // interleaved keys: a slot serves one tile at a time, released on bar_kv_empty[s]
                bool freed = true;
                if (!kPerTileMma || ilv || j < C::STAGES || j - C::STAGES < tile[0].nkv)
                    freed = mbar_wait(bar_kv_empty + s, ph ^ 1);
                if (kPerTileMma && !ilv && freed && (j < C::STAGES || j - C::STAGES < tile[1].nkv))
                    freed = mbar_wait(bar_kv_empty + C::STAGES + s, ph ^ 1);
                if (!freed) break;
                issued = j + 1;
                load_kv(j, pol_kv);
            }
            // no copy may still be landing in shared memory when the CTA exits
            mbar_wait(bar_q_full, 0);
            for (int j = issued - C::STAGES > 0 ? issued - C::STAGES : 0; j < issued; ++j) {
                mbar_wait(bar_k_full + j % C::STAGES, (j / C::STAGES) & 1);
                mbar_wait(bar_v_full + j % C::STAGES, (j / C::STAGES) & 1);
            }
        }
      } else if (C::EARLY && (warp == 1 || warp == 2)) {
        // =============================== MMA issuers (EARLY) ==============================
        // Warp 1 issues the MMAs of query tile 0, warp 2 those of tile 1 (one thread each).  Per
        // KV tile j: S_t(j+1) as soon as softmax t holds S_t(j) in registers (s_free_t), then
        // PV_t(j) per 64-key half of P_t(j) as the softmax hands it over (p_ready), then pv_done_t.
        // Each thread releases the stages its own tile used (a stage-release barrier per tile;
        // the producer waits for the tiles that used the stage).
        if (lane == 0) {
            const int t = warp - 1;
            const int nt = t ? tile[1].nkv : tile[0].nkv;
            constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, true);
            constexpr uint32_t hiK = desc_sw128_hi(1024);
            bool ok = mbar_wait(ROPE ? bar_q_ready : bar_q_full, 0);
            tc_fence_after();
            const uint32_t kvlo0 = desc_sw128_lo(smem_u32(sKV), 16);
            const uint32_t qlo = desc_sw128_lo(smem_u32(sQ + t * C::Q_TILES * C::TILE_BYTES), 16);
            const uint32_t dS = tmem + (t ? C::COL_S1 : C::COL_S0);
            const uint32_t dO = tmem + (t ? C::COL_O1 : C::COL_O0);
            const uint32_t aP = tmem + (t ? C::COL_P1 : C::COL_P0);
            auto issue_s = [&](int j) {
                const uint32_t klo = kvlo0 + ((ring_of(t, j) % C::STAGES) * C::STAGE_BYTES >> 4);
                constexpr int NCHAIN = ROPE ? 3 : 1;
#pragma unroll
                for (int ch = 0; ch < NCHAIN; ++ch) {
                    const uint32_t qa = qlo + (ch == 2 ? (C::TILE_BYTES >> 4) : 0);
                    const uint32_t kb = klo + (ch == 1 ? (C::TILE_BYTES >> 4) : 0);
#pragma unroll
                    for (int kk = 0; kk < C::KSTEPS; ++kk) {
                        constexpr uint32_t box16 = (C::TILE_BYTES / C::NBOX) >> 4;
                        const uint32_t off = (kk >> 2) * box16 + (kk & 3) * 2;
                        mma_ss(dS, desc_join(qa + off, hiK), desc_join(kb + off, hiK), idesc_qk,
                               (ch > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                mma_commit(bar_s_full + t);
            };
            auto issue_pv_half = [&](int j, int half) {
                const uint32_t va = smem_u32(sKV) + (ring_of(t, j) % C::STAGES) * C::STAGE_BYTES + C::K_TILES * C::TILE_BYTES;
                const uint32_t vlo = desc_sw128_lo(va, C::TILE_BYTES / C::NBOX);
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) {
                    const int kk = 4 * half + k4;
                    mma_ts(dO, aP + kk * 8, desc_join(vlo + kk * (2048 >> 4), hiK), idesc_pv,
                           (j > 0 || kk > 0) ? 1u : 0u);
                }
            };
            auto wait_k = [&](int j) {
                uint64_t* kb = ROPE == kRopeKFused ? bar_k_rot : bar_k_full;
                const int u = ring_of(t, j);
                const bool r = mbar_wait(kb + u % C::STAGES, (u / C::STAGES) & 1);
                tc_fence_after();
                return r;
            };
            if (ok && nt > 0) {
                ok = wait_k(0);
                if (ok) issue_s(0);
            }
            for (int j = 0; j < nkv; ++j) {
                const int u = ring_of(t, j), s = u % C::STAGES;
                if (j < nt) {
                    if (j + 1 < nt) {
                        if (ok) {
                            ok = mbar_wait(bar_s_free + t, j & 1);
                            tc_fence_after();
                        }
                        if (ok) ok = wait_k(j + 1);
                        if (ok) issue_s(j + 1);
                    }
                    if (ok) {
                        ok = mbar_wait(bar_v_full + s, (u / C::STAGES) & 1);
                        tc_fence_after();
                    }
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        if (ok) {
                            ok = mbar_wait(bar_p_ready + 2 * t + half, j & 1);
                            tc_fence_after();
                        }
                        if (ok) issue_pv_half(j, half);
                    }
                    mma_commit(bar_pv_done + t);
                    if (j == nt - 1) mma_commit(bar_o_done + t);
                    mma_commit(bar_kv_empty + (ilv ? 0 : t * C::STAGES) + s);   // this tile is done with stage s
                }
            }
            if (!ok) mma_commit(bar_o_done + t);
            mma_commit(bar_mma_final);
            mbar_wait(bar_mma_final, 0);
        }
      } else if (warp == 1 || (kOnesTwoIssuers && warp == 2)) {
        // =============================== MMA issuer(s) ===================================
        // kOnesTwoIssuers: warp 1 issues the MMAs of query tile 0, warp 2 those of tile 1, each
        // per KV tile j as  PV_t(j) first half, S_t(j+1), PV_t(j) second half  (P_SPLIT: the
        // second half of P_t(j) does not sit in S_t's columns), releasing its stages on a barrier
        // of its own (interleaved keys: the one of the slot, which serves one tile).
        // Otherwise one thread issues every MMA of both query tiles, interleaved per KV tile j as
        //   PV_0(j)  S_0(j+1)  PV_1(j)  S_1(j+1)
        // where S_t(j) = Q_t K_j^T (-> s_full_t) and PV_t(j): O_t += P_t(j) V_j.  The tensor core
        // runs one thread's MMAs in issue order, so S_t(j+1) overwrites the columns of P_t(j)
        // only after PV_t(j) has read them, and each softmax warpgroup works on its tile while
        // the tensor core runs the other tile's two products.  A commit signals the completion of
        // every MMA issued before it: s_full_t after S_t(j+1) therefore also means PV_t(j) is done,
        // so the softmax may correct O_t in place before it hands over P_t(j+1).
        // With a single K/V stage (D=128 with RoPE) S(j+1) has to wait for the stage to be
        // released after PV(j), so both tiles' S(j+1) follow the release.
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, C::N_PV, true);
            constexpr uint32_t hiK = desc_sw128_hi(1024);
            constexpr bool EARLY_S = C::STAGES > 1;
            const int nt0 = tile[0].nkv, nt1 = tile[1].nkv;
            bool ok = mbar_wait(ROPE ? bar_q_ready : bar_q_full, 0);
            tc_fence_after();
            // Descriptors: the high words are constants, the low words advance with the start
            // address (16-byte units), so an MMA costs one add and the instruction itself.
            const uint32_t kvlo0 = desc_sw128_lo(smem_u32(sKV), 16);
            // V of stage s: the second 64-wide N block is D's upper half (D=128) or the ones
            // block (D=64, leading-byte offset ones - V_s)
            auto v_lo = [&](int s) {
                const uint32_t va = smem_u32(sKV) + s * C::STAGE_BYTES + C::K_TILES * C::TILE_BYTES;
                return desc_sw128_lo(va, C::ONES ? smem_u32(sOnes) - va : C::TILE_BYTES / C::NBOX);
            };
            auto issue_s = [&](int t, int j) {
                const uint32_t qlo = desc_sw128_lo(smem_u32(sQ + t * C::Q_TILES * C::TILE_BYTES), 16);
                const uint32_t dS = tmem + (t ? C::COL_S1 : C::COL_S0);
                const uint32_t klo = kvlo0 + ((ring_of(t, j) % C::STAGES) * C::STAGE_BYTES >> 4);
                // chains: (Qh,Kh) [+ (Qh,Kl) + (Ql,Kh) with RoPE]
                constexpr int NCHAIN = ROPE ? 3 : 1;
#pragma unroll
                for (int ch = 0; ch < NCHAIN; ++ch) {
                    const uint32_t qa = qlo + (ch == 2 ? (C::TILE_BYTES >> 4) : 0);
                    const uint32_t kb = klo + (ch == 1 ? (C::TILE_BYTES >> 4) : 0);
#pragma unroll
                    for (int kk = 0; kk < C::KSTEPS; ++kk) {
                        // K step kk: box kk/4, 32-byte column offset (kk%4) inside the 128-byte row
                        constexpr uint32_t box16 = (C::TILE_BYTES / C::NBOX) >> 4;
                        const uint32_t off = (kk >> 2) * box16 + (kk & 3) * 2;
                        mma_ss(dS, desc_join(qa + off, hiK), desc_join(kb + off, hiK), idesc_qk,
                               (ch > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                mma_commit(bar_s_full + t);
            };
            // PV_t(j) for keys [64 half, 64 half + 64): issued as soon as the softmax has written
            // that half of P_t(j), so the product overlaps the exponentials of the other half
            auto issue_pv_half = [&](int t, int j, int half) {
                const uint32_t dO = tmem + (t ? C::COL_O1 : C::COL_O0);
                // P_SPLIT: the second half of P sits after O_t
                const uint32_t aP = (kPSplit && half) ? tmem + (t ? C::COL_PH1 : C::COL_PH0) - 32
                                                         : tmem + (t ? C::COL_S1 : C::COL_S0);
                const uint32_t vlo = v_lo(ring_of(t, j) % C::STAGES);
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) {
                    // keys [16kk, 16kk+16): 16 rows of 128 B in every 64-wide D box
                    const int kk = 4 * half + k4;
                    mma_ts(dO, aP + kk * 8, desc_join(vlo + kk * (2048 >> 4), hiK), idesc_pv,
                           (j > 0 || kk > 0) ? 1u : 0u);
                }
                if (kPSplit && half == 1) mma_commit(bar_pv_done + t);   // P_t's second half is free again
                if (half == 1 && j == (t ? nt1 : nt0) - 1) mma_commit(bar_o_done + t);
            };
            auto wait_k = [&](int u) {   // K of ring index u in place
                uint64_t* kb = ROPE == kRopeKFused ? bar_k_rot : bar_k_full;
                const bool r = mbar_wait(kb + u % C::STAGES, (u / C::STAGES) & 1);
                tc_fence_after();
                return r;
            };
            const int nkv_all = max(nt0, nt1);
            if constexpr (kOnesTwoIssuers) {
                const int t = warp - 1;
                const int n = t ? nt1 : nt0;
                if (ok && n > 0) {
                    ok = wait_k(ring_of(t, 0));
                    if (ok) issue_s(t, 0);
                }
                for (int j = 0; j < n; ++j) {
                    const int u = ring_of(t, j), s = u % C::STAGES;
                    if (ok) {
                        ok = mbar_wait(bar_v_full + s, (u / C::STAGES) & 1);
                        tc_fence_after();
                    }
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        if (ok) {
                            ok = mbar_wait(bar_p_ready + 2 * t + half, j & 1);
                            tc_fence_after();
                        }
                        if (ok) issue_pv_half(t, j, half);
                        // S_t(j+1) overwrites S_t: after the PV half that reads P from there
                        if (half == (kPSplit ? 0 : 1) && ok && j + 1 < n) {
                            ok = wait_k(ring_of(t, j + 1));
                            if (ok) issue_s(t, j + 1);
                        }
                    }
                    mma_commit(bar_kv_empty + (ilv ? 0 : t * C::STAGES) + s);   // this tile is done with stage s
                }
                if (!ok) mma_commit(bar_o_done + t);
            } else {
            if (ok && nkv_all > 0) {
                ok = wait_k(0);
                if (ok && nt0 > 0) issue_s(0, 0);
                if (ilv && ok && nt1 > 0) ok = wait_k(1);
                if (ok && nt1 > 0) issue_s(1, 0);
            }
            // Interleaved keys, per step j and tile t (ring index u = 2j + t):
            //   PV_t(j) from slot u, release of slot u, S_t(j+1) from slot u + 2
            for (int j = 0; ilv && j < nkv_all; ++j) {
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    const int n = t ? nt1 : nt0;
                    if (j >= n) continue;
                    const int u = 2 * j + t, s = u % C::STAGES;
                    if (ok) {
                        ok = mbar_wait(bar_v_full + s, (u / C::STAGES) & 1);
                        tc_fence_after();
                    }
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        if (ok) {
                            ok = mbar_wait(bar_p_ready + 2 * t + half, j & 1);
                            tc_fence_after();
                        }
                        if (ok) issue_pv_half(t, j, half);
                        // P_SPLIT: S_t(j+1) may follow the first half of PV_t(j)
                        if (half == (kPSplit ? 0 : 1) && ok && j + 1 < n) {
                            ok = wait_k(u + 2);
                            if (ok) issue_s(t, j + 1);
                        }
                    }
                    mma_commit(bar_kv_empty + s);
                }
            }
            for (int j = 0; !ilv && j < nkv_all; ++j) {
                const int s = j % C::STAGES;
                if (ok) {
                    ok = mbar_wait(bar_v_full + s, (j / C::STAGES) & 1);
                    tc_fence_after();
                }
                bool k_next = false;   // K(j+1) waited for
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    const int n = t ? nt1 : nt0;
                    if (j >= n) continue;
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        if (ok) {
                            ok = mbar_wait(bar_p_ready + 2 * t + half, j & 1);
                            tc_fence_after();
                        }
                        if (ok) issue_pv_half(t, j, half);
                        // P_SPLIT: S_t(j+1) may follow the first half of PV_t(j)
                        if (half == (kPSplit ? 0 : 1) && EARLY_S && ok && j + 1 < n) {
                            if (!k_next) ok = wait_k(j + 1);
                            k_next = true;
                            if (ok) issue_s(t, j + 1);
                        }
                    }
                }
                // stage s is free once every MMA issued so far has completed
                mma_commit(bar_kv_empty + s);
                if (!EARLY_S && ok && j + 1 < nkv_all) {
                    ok = wait_k(j + 1);
                    if (ok && j + 1 < nt0) issue_s(0, j + 1);
                    if (ok && j + 1 < nt1) issue_s(1, j + 1);
                }
            }
            // a tile whose pipeline stopped early still gets its completion signal
            if (!ok) {
                mma_commit(bar_o_done + 0);
                mma_commit(bar_o_done + 1);
            }
            }
            // every MMA issued above must be complete before tensor memory is released
            mma_commit(bar_mma_final);
            mbar_wait(bar_mma_final, 0);
        }
      } else if (C::MASK_SLOTS > 0 && (warp == 2 || warp == 3)) {
        // =============================== mask producers (MASK_TMA) ========================
        // Warp 2 loads the mask of query tile 0, warp 3 that of tile 1: per key tile of the
        // query tile, four 32-key x 128-row fp32 boxes in key order through the tile's
        // MASK_SLOTS slots (rows past Sq and keys past Skv arrive as zeros).  The mask is viewed
        // as [Bm][Hm][Sq][Skv] with Bm or Hm = 1 where it broadcasts.
        if constexpr (C::MASK_SLOTS > 0) if (lane == 0 && p.mask_tma) {
            const int t = warp - 2;
            const bool act = t ? tile[1].active : tile[0].active;
            const int nt = t ? tile[1].nkv : tile[0].nkv;
            const int r0 = t ? tile[1].r0 : tile[0].r0;
            const int hm = p.mask_hs ? (t ? tile[1].h : tile[0].h) : 0;
            const int bm = p.mask_bs ? b : 0;
            uint64_t* mfull = bar_m_full + t * C::MASK_SLOTS;
            uint64_t* mempty = bar_m_empty + t * C::MASK_SLOTS;
            uint8_t* mbase = sMask + t * C::MASK_SLOTS * C::MASK_BOX_BYTES;
            const uint64_t pol = l2_policy_evict_last();   // the mask is shared by every head it broadcasts to
            int issued = 0;
            bool okm = act;
            for (int j = 0; okm && j < nt; ++j) {
                const int k0 = (kv0 + ring_of(t, j)) * 128;
                for (int c = 0; c < 4; ++c) {
                    const int u = 4 * j + c, sl = u % C::MASK_SLOTS;
                    okm = mbar_wait(mempty + sl, ((u / C::MASK_SLOTS) & 1) ^ 1);
                    if (!okm) break;
                    mbar_arrive_expect_tx(mfull + sl, C::MASK_BOX_BYTES);
                    tma_load_4d(&tm_m, mfull + sl, mbase + sl * C::MASK_BOX_BYTES, k0 + 32 * c, r0, hm, bm, pol);
                    issued = u + 1;
                }
            }
            // no copy may still be landing in shared memory when the CTA exits
            for (int u = issued - C::MASK_SLOTS > 0 ? issued - C::MASK_SLOTS : 0; u < issued; ++u)
                mbar_wait(mfull + u % C::MASK_SLOTS, (u / C::MASK_SLOTS) & 1);
        }
      } else if (ROPE == kRopeKFused) {
        // =============================== K rotation (warps 2, 3) ========================
        // Each K tile is rotated in place as soon as it lands: key r of the tile (position
        // (kv0 + j) * 128 + r, as for the pre-rotated form) is split into hi = bf16(k') in the Kh
        // slot and lo = bf16(k' - hi) in the Kl slot; thread u handles keys u, u + NROT, ....  The
        // pairs (2i, 2i+1) share a 16-byte chunk, which the 128-byte swizzle moves whole.
        constexpr int NROT = C::EARLY ? 32 : 64;   // warp 3 alone when warp 2 issues MMAs
        const int u = C::EARLY ? lane : (warp - 2) * 32 + lane;
        for (int j = 0; j < n_loads; ++j) {   // j: ring index = key tile kv0 + j
            const int s = j % C::STAGES;
            if (!mbar_wait(bar_k_full + s, (j / C::STAGES) & 1)) break;
            uint8_t* kh = sKV + s * C::STAGE_BYTES;
            uint8_t* kl = kh + C::TILE_BYTES;
#pragma unroll
            for (int rr = 0; rr < 128 / NROT; ++rr) {
                const int r = u + NROT * rr;
                const long pos = static_cast<long>(kv0 + j) * 128 + r;
                if (pos < p.Skv) {
                    const float4* tab4 = reinterpret_cast<const float4*>(p.rope_tab + pos * (D / 2));
#pragma unroll 1
                    for (int bx = 0; bx < C::NBOX; ++bx) {
#pragma unroll 2
                        for (int ck = 0; ck < 8; ++ck) {
                            const uint32_t o = bx * (C::TILE_BYTES / C::NBOX) + sw128_offset(r, ck);
                            const uint4 w = *reinterpret_cast<const uint4*>(kh + o);
                            const float4 c01 = __ldg(tab4 + bx * 16 + ck * 2);
                            const float4 c23 = __ldg(tab4 + bx * 16 + ck * 2 + 1);
                            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
                            const float2 cs[4] = {make_float2(c01.x, c01.y), make_float2(c01.z, c01.w),
                                                  make_float2(c23.x, c23.y), make_float2(c23.z, c23.w)};
                            uint32_t hh[4], ll[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float x0 = bf16lo_to_f32(ww[e]), x1 = bf16hi_to_f32(ww[e]);
                                const float y0 = x0 * cs[e].x - x1 * cs[e].y;
                                const float y1 = x0 * cs[e].y + x1 * cs[e].x;
                                hh[e] = pack_bf16x2(y0, y1);
                                ll[e] = pack_bf16x2(y0 - bf16lo_to_f32(hh[e]), y1 - bf16hi_to_f32(hh[e]));
                            }
                            *reinterpret_cast<uint4*>(kh + o) = make_uint4(hh[0], hh[1], hh[2], hh[3]);
                            *reinterpret_cast<uint4*>(kl + o) = make_uint4(ll[0], ll[1], ll[2], ll[3]);
                        }
                    }
                } else {
                    // keys past Skv: TMA zero-filled Kh; Kl gets zeros too
#pragma unroll
                    for (int bx = 0; bx < C::NBOX; ++bx)
#pragma unroll
                        for (int ck = 0; ck < 8; ++ck)
                            *reinterpret_cast<uint4*>(kl + bx * (C::TILE_BYTES / C::NBOX) + sw128_offset(r, ck)) =
                                make_uint4(0, 0, 0, 0);
                }
            }
            fence_proxy_async_smem();   // generic-proxy writes -> the tensor core's reads
            mbar_arrive(bar_k_rot + s);
        }
      }
    } else {
        setmaxnreg_inc<kRegsSoftmax>();
        // =============================== softmax warpgroups =============================
        const int wg = (warp - 4) >> 2;             // query tile index
        const int row = (warp & 3) * 32 + lane;     // 0..127 == TMEM lane
        TcTile T;
        T.h = wg ? tile[1].h : tile[0].h;
        T.r0 = wg ? tile[1].r0 : tile[0].r0;
        T.nkv = wg ? tile[1].nkv : tile[0].nkv;
        T.active = wg ? tile[1].active : tile[0].active;
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_base + (wg ? C::COL_S1 : C::COL_S0);
        const uint32_t tO = tmem + lane_base + (wg ? C::COL_O1 : C::COL_O0);
        const int qrow = T.r0 + row;                // absolute query row
        const long off_c = static_cast<long>(p.Skv) - p.Sq;
        bool ok = true;

        if (ROPE) {
            // rotate this row of the query tile in place: hi half -> Qh, remainder -> Ql
            ok = mbar_wait(bar_q_full, 0);
            if (ok && T.active && qrow < p.Sq) {
                uint8_t* qh = sQ + wg * C::Q_TILES * C::TILE_BYTES;
                uint8_t* ql = qh + C::TILE_BYTES;
                const float2* tab = p.rope_tab + static_cast<long>(p.q_pos0 + qrow) * (D / 2);
#pragma unroll
                for (int bx = 0; bx < C::NBOX; ++bx) {
#pragma unroll
                    for (int ck = 0; ck < 8; ++ck) {
                        const uint32_t o = bx * (C::TILE_BYTES / C::NBOX) + sw128_offset(row, ck);
                        uint4 w = *reinterpret_cast<uint4*>(qh + o);
                        uint32_t ww[4] = {w.x, w.y, w.z, w.w}, hh[4], ll[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 cs = tab[bx * 32 + ck * 4 + e];
                            const float x0 = bf16lo_to_f32(ww[e]), x1 = bf16hi_to_f32(ww[e]);
                            const float y0 = x0 * cs.x - x1 * cs.y;
                            const float y1 = x0 * cs.y + x1 * cs.x;
                            hh[e] = pack_bf16x2(y0, y1);
                            ll[e] = pack_bf16x2(y0 - bf16lo_to_f32(hh[e]), y1 - bf16hi_to_f32(hh[e]));
                        }
                        *reinterpret_cast<uint4*>(qh + o) = make_uint4(hh[0], hh[1], hh[2], hh[3]);
                        *reinterpret_cast<uint4*>(ql + o) = make_uint4(ll[0], ll[1], ll[2], ll[3]);
                    }
                }
            } else if (ok && T.active) {
                // rows past Sq were zero-filled by TMA; give Ql zeros too
                uint8_t* ql = sQ + wg * C::Q_TILES * C::TILE_BYTES + C::TILE_BYTES;
#pragma unroll
                for (int bx = 0; bx < C::NBOX; ++bx)
#pragma unroll
                    for (int ck = 0; ck < 8; ++ck)
                        *reinterpret_cast<uint4*>(ql + bx * (C::TILE_BYTES / C::NBOX) + sw128_offset(row, ck)) =
                            make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
            mbar_arrive(bar_q_ready);
        }

        float m_run = -INFINITY;   // running max used in the exponent (log2 units)
        float l_run = 0.f;         // row sum of the fp32 weights (logsumexp)
        float l_mma = 0.f;         // row sum of the bf16-rounded weights (normalises O)
        const float sl2 = p.scale_log2;
        const uint32_t tP = tS;    // P_t(j) is written over the first 64 columns of S_t ...
        // ... or, P_SPLIT, its keys [64, 128) after O_t
        const uint32_t tPh = tmem + lane_base + (wg ? C::COL_PH1 : C::COL_PH0);
        if constexpr (C::EARLY) {
        // Exponentiation turns: warpgroup 0 exponentiates, then warpgroup 1, alternately; each
        // group's loads, row max, stores and hand-offs overlap the other group's exponentials.
        // Both groups walk every key tile of the CTA (a tile past its own end only passes the
        // barriers), so the turn phases match.  Without a second active tile there are no turns.
        const bool turns = tile[0].active && tile[1].active;
        const int nsteps = turns ? nkv : T.nkv;
        const uint32_t tP = tmem + lane_base + (wg ? C::COL_P1 : C::COL_P0);
        for (int j = 0; j < nsteps; ++j) {
            const bool mine = j < T.nkv;
            uint32_t sr[4][32];
            if (mine) {
                if (ok && !__all_sync(0xffffffffu, mbar_wait(bar_s_full + wg, j & 1))) ok = false;
                tc_fence_after();
            }
            const bool go = mine && ok;
            if (go) {
#pragma unroll
                for (int cb = 0; cb < 4; ++cb) tmem_ld32(tS + cb * 32, sr[cb]);
                tmem_wait_ld();
            }
            if (mine) {
                // S_t(j) is in registers: the MMA thread may compute S_t(j+1) into its columns
                tc_fence_before();
                mbar_arrive(bar_s_free + wg);
            }
            bool need = false;
            float corr = 1.f;
            if (go) {
            const int k0 = (kv0 + ring_of(wg, j)) * 128;
                if (MASK && qrow < p.Sq) {
                    // additive mask: S holds q.k unscaled, so add mask / scale; the exponent
                    // (s * scale + mask) * log2(e) - m then keeps its form
                    const float* mrow = p.mask + b * p.mask_bs + T.h * p.mask_hs + static_cast<long>(qrow) * p.Skv + k0;
                    const int ncol = p.Skv - k0;
                    if (p.mask_vec4 && ncol >= 128) {
                        // 16-byte loads (mask rows 16-byte aligned): a quarter of the L1 wavefronts
#pragma unroll
                        for (int cb = 0; cb < 4; ++cb)
#pragma unroll
                            for (int e4 = 0; e4 < 8; ++e4) {
                                const float4 m4 = __ldg(reinterpret_cast<const float4*>(mrow + cb * 32 + 4 * e4));
                                const float mm[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
                                for (int u = 0; u < 4; ++u)
                                    sr[cb][4 * e4 + u] = __float_as_uint(__uint_as_float(sr[cb][4 * e4 + u]) + mm[u] * p.inv_scale);
                            }
                    } else {
#pragma unroll
                        for (int cb = 0; cb < 4; ++cb)
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                if (cb * 32 + e < ncol)
                                    sr[cb][e] = __float_as_uint(__uint_as_float(sr[cb][e]) + __ldg(mrow + cb * 32 + e) * p.inv_scale);
                    }
                }
                // mask: keys past Skv, and (causal) keys beyond this row's diagonal
                const long lim_causal = p.causal ? static_cast<long>(qrow) + off_c : static_cast<long>(p.Skv) - 1;
                const long lim = lim_causal < p.Skv - 1 ? lim_causal : static_cast<long>(p.Skv) - 1;
                float mx = -INFINITY;
                if (static_cast<long>(k0) + 127 > lim) {
                    const long nvis = lim - k0 + 1;     // keys [k0, k0+nvis) visible
#pragma unroll
                    for (int cb = 0; cb < 4; ++cb)
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (cb * 32 + e >= nvis) sr[cb][e] = __float_as_uint(-INFINITY);
                }
                {
                    // eight independent three-input max chains, then a short tree
                    float mp[8];
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint32_t* r = &sr[c >> 1][(c & 1) * 16];
                        float a = fmaxf(__uint_as_float(r[0]), __uint_as_float(r[1]));
#pragma unroll
                        for (int e = 2; e < 16; e += 2) a = max3(a, __uint_as_float(r[e]), __uint_as_float(r[e + 1]));
                        mp[c] = a;
                    }
                    mx = max3(max3(mp[0], mp[1], mp[2]), max3(mp[3], mp[4], mp[5]), fmaxf(mp[6], mp[7]));
                }
                const float tmax = mx * sl2;
                need = tmax > m_run + kRescaleThreshold;
                if (need) {
                    corr = (m_run == -INFINITY) ? 0.f : fast_exp2(m_run - tmax);
                    m_run = tmax;
                }
                l_run *= corr;
                l_mma *= corr;
                // P_t and O_t are free once PV_t(j-1) completed (issued when P_t(j-1) was handed
                // over, long done by now); O is corrected before PV_t(j) may start
                if (j > 0) {
                    if (!__all_sync(0xffffffffu, mbar_wait(bar_pv_done + wg, (j - 1) & 1))) ok = false;
                    tc_fence_after();
                    if (__any_sync(0xffffffffu, need)) {
#pragma unroll
                        for (int ob = 0; ob < D / 16; ++ob) {
                            uint32_t orr[16];
                            tmem_ld16(tO + ob * 16, orr);
                            tmem_wait_ld();
#pragma unroll
                            for (int e = 0; e < 16; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * corr);
                            tmem_st16(tO + ob * 16, orr);
                        }
                    }
                }
            }
            if (turns) {
                if (wg == 0) {
                    if (j > 0) named_bar_sync(kTcBarTurn1, 256);
                } else {
                    named_bar_sync(kTcBarTurn0, 256);
                }
            }
            if (go) {
                const float mu = (m_run == -INFINITY) ? 0.f : m_run;
                uint64_t lt2[4] = {0, 0, 0, 0}, lr2[4] = {0, 0, 0, 0};
                const uint64_t sl2x2 = f2_pack(sl2, sl2);
                const uint64_t nmux2 = f2_pack(-mu, -mu);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int cb = 2 * half + u;
                        uint32_t pk[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            float t0, t1;
                            f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[cb][2 * e]), __uint_as_float(sr[cb][2 * e + 1])),
                                             sl2x2, nmux2),
                                      t0, t1);
                            const float p0 = fast_exp2(t0);
                            const float p1 = fast_exp2(t1);
                            lt2[e & 3] = f2_add(lt2[e & 3], f2_pack(p0, p1));
                            pk[e] = pack_bf16x2(p0, p1);
                            lr2[e & 3] = f2_add(lr2[e & 3], f2_pack(bf16lo_to_f32(pk[e]), bf16hi_to_f32(pk[e])));
                        }
                        if (cb == 3) {
                            // the exponentials are done: the other group's turn
                            if (turns && wg == 0)
                                named_bar_arrive(kTcBarTurn0, 256);
                            else if (turns && j + 1 < nkv)
                                named_bar_arrive(kTcBarTurn1, 256);
                        }
                        tmem_st16(tP + cb * 16, pk);
                    }
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(bar_p_ready + 2 * wg + half);
                }
                float a, c;
                f2_unpack(f2_add(f2_add(lt2[0], lt2[1]), f2_add(lt2[2], lt2[3])), a, c);
                l_run += a + c;
                f2_unpack(f2_add(f2_add(lr2[0], lr2[1]), f2_add(lr2[2], lr2[3])), a, c);
                l_mma += a + c;
            } else {
                if (turns) {
                    if (wg == 0)
                        named_bar_arrive(kTcBarTurn0, 256);
                    else if (j + 1 < nkv)
                        named_bar_arrive(kTcBarTurn1, 256);
                }
                if (mine) {
                    // keep the MMA thread's counts; it stops on its own
                    mbar_arrive(bar_p_ready + 2 * wg);
                    mbar_arrive(bar_p_ready + 2 * wg + 1);
                }
            }
        }
        } else {
        for (int j = 0; j < T.nkv; ++j) {
            uint32_t sr[4][32];
            if (ok && !__all_sync(0xffffffffu, mbar_wait(bar_s_full + wg, j & 1))) ok = false;
            tc_fence_after();
            if (!ok) {
                // keep the MMA thread's counts; it stops on its own
                mbar_arrive(bar_p_ready + 2 * wg);
                mbar_arrive(bar_p_ready + 2 * wg + 1);
                continue;
            }
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) tmem_ld32(tS + cb * 32, sr[cb]);
            tmem_wait_ld();
            const int k0 = (kv0 + ring_of(wg, j)) * 128;
            if (C::MASK_SLOTS > 0 && p.mask_tma) {
                // additive mask from the tile's slots: box c holds keys [32c, 32c+32) of all 128
                // rows, 16-byte chunk e of row r at chunk e ^ (r & 7) (the load's 128-byte
                // swizzle), so the row-per-thread reads are free of bank conflicts; S holds q.k
                // unscaled, so the mask enters as mask / scale
                const uint8_t* mrow = sMask + wg * C::MASK_SLOTS * C::MASK_BOX_BYTES + row * 128;
#pragma unroll
                for (int cb = 0; cb < 4; ++cb) {
                    constexpr int MS = C::MASK_SLOTS > 0 ? C::MASK_SLOTS : 1;   // (kernels without the ring never get here)
                    const int u = 4 * j + cb, sl = u % MS;
                    if (ok && !__all_sync(0xffffffffu, mbar_wait(bar_m_full + wg * C::MASK_SLOTS + sl, (u / MS) & 1)))
                        ok = false;
                    const uint8_t* mb = mrow + sl * C::MASK_BOX_BYTES;
#pragma unroll
                    for (int e4 = 0; e4 < 8; ++e4) {
                        const float4 m4 = *reinterpret_cast<const float4*>(mb + ((e4 ^ (row & 7)) << 4));
                        const float mm[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4)
                            sr[cb][4 * e4 + q4] = __float_as_uint(__uint_as_float(sr[cb][4 * e4 + q4]) + mm[q4] * p.inv_scale);
                    }
                    // the slot may be refilled: this thread's generic-proxy reads of it are ordered
                    // before the next TMA (async-proxy) write into it
                    fence_proxy_async_smem();
                    mbar_arrive(bar_m_empty + wg * C::MASK_SLOTS + sl);
                }
            } else if (MASK && qrow < p.Sq) {
                // additive mask: S holds q.k unscaled, so add mask / scale; the exponent
                // (s * scale + mask) * log2(e) - m then keeps its form
                const float* mrow = p.mask + b * p.mask_bs + T.h * p.mask_hs + static_cast<long>(qrow) * p.Skv + k0;
                const int ncol = p.Skv - k0;
                if (p.mask_vec4 && ncol >= 128) {
                    // 16-byte loads (mask rows 16-byte aligned): a quarter of the L1 wavefronts
#pragma unroll
                    for (int cb = 0; cb < 4; ++cb)
#pragma unroll
                        for (int e4 = 0; e4 < 8; ++e4) {
                            const float4 m4 = __ldg(reinterpret_cast<const float4*>(mrow + cb * 32 + 4 * e4));
                            const float mm[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
                            for (int u = 0; u < 4; ++u)
                                sr[cb][4 * e4 + u] = __float_as_uint(__uint_as_float(sr[cb][4 * e4 + u]) + mm[u] * p.inv_scale);
                        }
                } else {
#pragma unroll
                    for (int cb = 0; cb < 4; ++cb)
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (cb * 32 + e < ncol)
                                sr[cb][e] = __float_as_uint(__uint_as_float(sr[cb][e]) + __ldg(mrow + cb * 32 + e) * p.inv_scale);
                }
            }
            // mask: keys past Skv, and (causal) keys beyond this row's diagonal
            const long lim_causal = p.causal ? static_cast<long>(qrow) + off_c : static_cast<long>(p.Skv) - 1;
            const long lim = lim_causal < p.Skv - 1 ? lim_causal : static_cast<long>(p.Skv) - 1;
            float mx = -INFINITY;
            if (static_cast<long>(k0) + 127 > lim) {
                const long nvis = lim - k0 + 1;     // keys [k0, k0+nvis) visible
#pragma unroll
                for (int cb = 0; cb < 4; ++cb)
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (cb * 32 + e >= nvis) sr[cb][e] = __float_as_uint(-INFINITY);
            }
            {
                // eight independent three-input max chains, then a short tree
                float mp[8];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint32_t* r = &sr[c >> 1][(c & 1) * 16];
                    float a = fmaxf(__uint_as_float(r[0]), __uint_as_float(r[1]));
#pragma unroll
                    for (int e = 2; e < 16; e += 2) a = max3(a, __uint_as_float(r[e]), __uint_as_float(r[e + 1]));
                    mp[c] = a;
                }
                mx = max3(max3(mp[0], mp[1], mp[2]), max3(mp[3], mp[4], mp[5]), fmaxf(mp[6], mp[7]));
            }
            const float tmax = mx * sl2;
            // lazy rescale: move the exponent's max only when the block max exceeds it by > threshold
            const bool need = tmax > m_run + kRescaleThreshold;
            float corr = 1.f;
            if (need) {
                corr = (m_run == -INFINITY) ? 0.f : fast_exp2(m_run - tmax);
                m_run = tmax;
            }
            // O correction, only in warps with a rescaling row and once O holds earlier blocks.
            // PV_t(j) is issued only after this warpgroup's p_ready arrivals below; PV_t(j-1) had
            // completed before s_full_t(j) was signalled, except (P_SPLIT) its second half, which
            // follows S_t(j) and is waited for here (and before the second half of P_t(j) takes
            // its columns).
            bool pv_prev = !(kPSplit && j > 0);   // PV_t(j-1) known complete
            auto wait_pv_prev = [&]() {
                if (ok && !__all_sync(0xffffffffu, mbar_wait(bar_pv_done + wg, (j - 1) & 1))) ok = false;
                tc_fence_after();
                pv_prev = true;
            };
            if (j > 0 && __any_sync(0xffffffffu, need)) {
                if (!pv_prev) wait_pv_prev();
#pragma unroll
                for (int cb = 0; cb < (C::N_PV + 31) / 32; ++cb) {
                    uint32_t orr[32];
                    tmem_ld32(tO + cb * 32, orr);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * corr);
                    tmem_st32(tO + cb * 32, orr);
                }
            }
            l_run *= corr;
            l_mma *= corr;
            const float mu = (m_run == -INFINITY) ? 0.f : m_run;
            // p = exp2(s*scale*log2e - mu) in fp32, rounded to bf16 for the PV MMA.  Two row sums:
            // the exact one (for the logsumexp) and the sum of the rounded values the MMA uses
            // (O is normalised by it, so the rounding of a dominant weight cancels).
            uint64_t lt2[4] = {0, 0, 0, 0}, lr2[4] = {0, 0, 0, 0};   // packed partial sums, 4 chains each
            const uint64_t sl2x2 = f2_pack(sl2, sl2);
            const uint64_t nmux2 = f2_pack(-mu, -mu);
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) {
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    float t0, t1;
                    f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[cb][2 * e]), __uint_as_float(sr[cb][2 * e + 1])),
                                     sl2x2, nmux2),
                              t0, t1);
                    const float p0 = fast_exp2(t0);
                    const float p1 = fast_exp2(t1);
                    lt2[e & 3] = f2_add(lt2[e & 3], f2_pack(p0, p1));
                    pk[e] = pack_bf16x2(p0, p1);
                    if (!C::ONES)
                        lr2[e & 3] = f2_add(lr2[e & 3], f2_pack(bf16lo_to_f32(pk[e]), bf16hi_to_f32(pk[e])));
                }
                if (kPSplit && cb == 2 && !pv_prev) wait_pv_prev();
                tmem_st16((kPSplit && cb >= 2) ? tPh + (cb - 2) * 16 : tP + cb * 16, pk);
                if (cb == 1) {
                    // keys [0, 64) of P are in TMEM: the first half of PV may start
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(bar_p_ready + 2 * wg);
                }
            }
            {
                float a, c;
                f2_unpack(f2_add(f2_add(lt2[0], lt2[1]), f2_add(lt2[2], lt2[3])), a, c);
                l_run += a + c;
                if (!C::ONES) {
                    f2_unpack(f2_add(f2_add(lr2[0], lr2[1]), f2_add(lr2[2], lr2[3])), a, c);
                    l_mma += a + c;
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar_p_ready + 2 * wg + 1);
        }

        }
        // Epilogue: O / l -> bf16 or fp32, and the logsumexp.  With interleaved keys the two
        // warpgroups hold partial states (m_t, l_t, O_t) of the same rows: they exchange m and
        // the row sums through shared memory (each in its own Q slot, free once its products are
        // done) and each writes half of the columns of the merged
        //   O = (a_0 O_0 + a_1 O_1) / (a_0 l_0 + a_1 l_1),  a_t = 2^(m_t - max(m_0, m_1)).
        // The TMEM reads are warp-collective, so every lane of the warp takes part; only rows
        // inside [0, Sq) are stored.
        if (T.active) {
            bool have = ok && T.nkv > 0;   // warp-uniform: this tile's O holds products
            if (have) {
                have = __all_sync(0xffffffffu, mbar_wait(bar_o_done + wg, 0));
                tc_fence_after();
            } else if (ilv) {
                // the merge below writes to the Q slot: its copy must have landed (no product
                // waited for it) ...
                mbar_wait(bar_q_full, 0);
            }
            // ... and with RoPE every row of it must be rotated: without a product of this tile
            // nothing has ordered the other rows' rotation before this point (T.nkv is uniform
            // over the warpgroup, so all of its threads meet here)
            if (ilv && ROPE && T.nkv == 0) {
                if (wg == 0)
                    named_bar_sync(kTcBarGroup0, 128);
                else
                    named_bar_sync(kTcBarGroup0 + 1, 128);
            }
            const bool store = qrow < p.Sq;
            if (C::ONES && have) {
                // the row sum of the rounded weights, accumulated by the PV MMA in column D of O
                uint32_t sr1[32];
                tmem_ld32(tO + D, sr1);
                tmem_wait_ld();
                l_mma = __uint_as_float(sr1[0]);
            }
            float m_fin = m_run;                      // exponent base of the result
            float l_fin = have ? l_run : 0.f;         // exact row sum (logsumexp)
            float lm_fin = have ? l_mma : 0.f;        // row sum of the rounded weights (normalises O)
            float a_own = 1.f, a_oth = 0.f;           // weights of this tile's O and the other's
            bool oth = false;                         // warp-uniform: the other tile's O is read too
            uint32_t tO_oth = 0;
            if (ilv) {
                const bool valid = have && l_run > 0.f;
                const float m_own = valid ? m_run : -INFINITY;
                float* xs = reinterpret_cast<float*>(sQ + wg * C::Q_TILES * C::TILE_BYTES);
                const float* xo = reinterpret_cast<const float*>(sQ + (1 - wg) * C::Q_TILES * C::TILE_BYTES);
                xs[row] = m_own;
                xs[128 + row] = l_run;
                xs[256 + row] = l_mma;
                named_bar_sync(kTcBarMerge, 256);
                tc_fence_after();   // the other group's o_done wait orders the reads of its O
                const float m_o = xo[row], lr_o = xo[128 + row], lm_o = xo[256 + row];
                m_fin = fmaxf(m_own, m_o);
                a_own = valid ? fast_exp2(m_own - m_fin) : 0.f;
                a_oth = m_o != -INFINITY ? fast_exp2(m_o - m_fin) : 0.f;
                l_fin = (valid ? a_own * l_run : 0.f) + (m_o != -INFINITY ? a_oth * lr_o : 0.f);
                lm_fin = (valid ? a_own * l_mma : 0.f) + (m_o != -INFINITY ? a_oth * lm_o : 0.f);
                oth = __any_sync(0xffffffffu, m_o != -INFINITY);
                tO_oth = tmem + lane_base + (wg ? C::COL_O0 : C::COL_O1);
            }
            const float inv = lm_fin > 0.f ? 1.f / lm_fin : 0.f;
            // a key split writes its normalised partial O (fp32) and its logsumexp to its slabs
            float* out_f32 = p.o_f32;
            __nv_bfloat16* out_bf16 = p.o;
            float* out_lse = p.lse;
            if (p.kv_splits > 1) {
                const long rows = static_cast<long>(p.B) * p.Sq * p.Hq;
                out_f32 = p.o_part + split * rows * D;
                out_bf16 = nullptr;
                out_lse = p.lse_part + split * rows;
            }
            // Each thread stores its own row, 16 bytes per instruction.  (Staging the rows in
            // shared memory for whole-segment stores measured slower on B200 except for the fp32
            // partials of key splits.)  With interleaved keys warpgroup t writes columns
            // [t D/2, (t+1) D/2) of the merged O.
            if constexpr (ilv) {
                // Interleaved keys (D = 64): warpgroup t's half of the output, 32 columns of the
                // tile's 128 rows, leaves through one TMA store.  Each thread writes its row into
                // a box in the K/V ring (free: both tiles' products are done) in the store's
                // swizzled layout -- 16-byte chunk c of row r at chunk c ^ (r & 7) of a 128-byte
                // row (fp32), or c ^ ((r >> 1) & 3) of a 64-byte row (bf16) -- which keeps the
                // row-per-thread writes free of bank conflicts; rows past Sq are clipped by the
                // store.  (Direct stores from the threads touch a different line per lane.)
                static_assert(D == 64, "interleaved keys: one 32-column block per warpgroup");
                uint32_t orr[32], oro[32];
                if (have) tmem_ld32(tO + wg * 32, orr);
                if (oth) tmem_ld32(tO_oth + wg * 32, oro);
                if (have || oth) tmem_wait_ld();
                float v[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const float x = have ? a_own * __uint_as_float(orr[e]) : 0.f;
                    v[e] = (oth ? fmaf(a_oth, __uint_as_float(oro[e]), x) : x) * inv;
                }
                uint8_t* box = sKV + wg * 16384;   // 1024-byte aligned
                if (out_f32) {
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        *reinterpret_cast<float4*>(box + row * 128 + ((c ^ (row & 7)) << 4)) =
                            make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
                } else {
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        *reinterpret_cast<uint4*>(box + row * 64 + ((c ^ ((row >> 1) & 3)) << 4)) =
                            make_uint4(pack_bf16x2(v[8 * c], v[8 * c + 1]), pack_bf16x2(v[8 * c + 2], v[8 * c + 3]),
                                       pack_bf16x2(v[8 * c + 4], v[8 * c + 5]), pack_bf16x2(v[8 * c + 6], v[8 * c + 7]));
                }
                fence_proxy_async_smem();
                if (wg == 0)
                    named_bar_sync(kTcBarGroup0, 128);
                else
                    named_bar_sync(kTcBarGroup0 + 1, 128);
                if (row == 0) {
                    // the map covers [B'][Sq][Hq][D] with B' = kv_splits * B: split s, batch b at s B + b
                    tma_store_4d(&tm_o, box, wg * 32, T.h, T.r0, (p.kv_splits > 1 ? split * p.B : 0) + b);
                    tma_store_commit();
                    tma_store_wait_all();
                }
            }
            const long orow_off = ((static_cast<long>(b) * p.Sq + qrow) * p.Hq + T.h) * D;
#pragma unroll
            for (int ci = 0; ci < D / 32; ++ci) {
                if (ilv) break;
                const int cb = ci;
                uint32_t orr[32], oro[32];
                if (have) tmem_ld32(tO + cb * 32, orr);
                if (oth) tmem_ld32(tO_oth + cb * 32, oro);
                if (have || oth) tmem_wait_ld();
                float v[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const float x = have ? a_own * __uint_as_float(orr[e]) : 0.f;
                    v[e] = (oth ? fmaf(a_oth, __uint_as_float(oro[e]), x) : x) * inv;
                }
                if (!store) continue;
                if (out_f32) {
                    float4* dst = reinterpret_cast<float4*>(out_f32 + orow_off + cb * 32);
#pragma unroll
                    for (int e = 0; e < 8; ++e) dst[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
                } else {
                    uint4* dst = reinterpret_cast<uint4*>(out_bf16 + orow_off + cb * 32);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        dst[e] = make_uint4(pack_bf16x2(v[8 * e], v[8 * e + 1]), pack_bf16x2(v[8 * e + 2], v[8 * e + 3]),
                                            pack_bf16x2(v[8 * e + 4], v[8 * e + 5]), pack_bf16x2(v[8 * e + 6], v[8 * e + 7]));
                }
            }
            if (store && out_lse != nullptr && (!ilv || wg == 0))
                out_lse[(static_cast<long>(b) * p.Hq + T.h) * p.Sq + qrow] =
                    l_fin > 0.f ? (m_fin + fast_log2(l_fin)) * kLn2 : -INFINITY;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// Merge of a key-split forward: one warp per (b, query row, q head) combines the row's
// kv_splits partials by their logsumexp, as the split-KV decode does (oxibonsai-model 0.1.4
// src/layers/flash_decode.rs, combine_tile_outputs):  L = log sum_s e^(lse_s);
// O = sum_s e^(lse_s - L) o_s.
// Partials with lse_s = -inf (no visible key in that chunk) weigh nothing; a row with none at all
// gets O = 0 and LSE = -inf.  Launched as a programmatic dependent of the split forward.
constexpr int kPcThreads = 256;
constexpr int kMaxKvSplits = 16;   // <= 32: one split per lane for the logsumexp reduction

template <int D>
__global__ void __launch_bounds__(kPcThreads) prefill_combine_kernel(
    const float* __restrict__ o_part, const float* __restrict__ lse_part, __nv_bfloat16* __restrict__ o,
    float* __restrict__ o_f32, float* __restrict__ lse, int B, int Sq, int Hq, int nsplit) {
    constexpr int E = D / 32;   // output elements per lane
    griddep_wait();
    const long rows = static_cast<long>(B) * Sq * Hq;
    const long r = static_cast<long>(blockIdx.x) * (kPcThreads / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (r >= rows) return;   // whole warps leave together
    const int h = static_cast<int>(r % Hq);
    const long bq = r / Hq;
    const int qi = static_cast<int>(bq % Sq);
    const int b = static_cast<int>(bq / Sq);
    const long lrow = (static_cast<long>(b) * Hq + h) * Sq + qi;
    // Every load of the row is issued before any result is used (one round trip): the lse of
    // split `lane`, and this lane's slice of every split's partial (the partials of rows below
    // Sq are always written, zeros where a split saw no key, so all of them are finite).
    const float ls = lane < nsplit ? lse_part[lane * rows + lrow] : -INFINITY;
    float x[kMaxKvSplits][E];
#pragma unroll
    for (int sp = 0; sp < kMaxKvSplits; ++sp) {
        if (sp < nsplit) {
            const float* src = o_part + (sp * rows + r) * D + lane * E;
            if constexpr (E == 2) {
                const float2 v = *reinterpret_cast<const float2*>(src);
                x[sp][0] = v.x, x[sp][1] = v.y;
            } else {
                const float4 v = *reinterpret_cast<const float4*>(src);
                x[sp][0] = v.x, x[sp][1] = v.y, x[sp][2] = v.z, x[sp][3] = v.w;
            }
        } else {
#pragma unroll
            for (int e = 0; e < E; ++e) x[sp][e] = 0.f;
        }
    }
    float M = ls;
#pragma unroll
    for (int w = 16; w >= 1; w >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, w));
    const float wt = (M == -INFINITY || ls == -INFINITY) ? 0.f : __expf(ls - M);
    float total = wt;
#pragma unroll
    for (int w = 16; w >= 1; w >>= 1) total += __shfl_xor_sync(0xffffffffu, total, w);
    float acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
#pragma unroll
    for (int sp = 0; sp < kMaxKvSplits; ++sp) {
        const float ws = __shfl_sync(0xffffffffu, wt, sp);   // 0 for sp >= nsplit
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = fmaf(ws, x[sp][e], acc[e]);
    }
    const float inv = total > 0.f ? 1.f / total : 0.f;
    const long dst = r * D + lane * E;
    if constexpr (E == 2) {
        if (o_f32 != nullptr)
            *reinterpret_cast<float2*>(o_f32 + dst) = make_float2(acc[0] * inv, acc[1] * inv);
        else
            *reinterpret_cast<uint32_t*>(o + dst) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
    } else {
        if (o_f32 != nullptr)
            *reinterpret_cast<float4*>(o_f32 + dst) =
                make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
        else
            *reinterpret_cast<uint2*>(o + dst) =
                make_uint2(pack_bf16x2(acc[0] * inv, acc[1] * inv), pack_bf16x2(acc[2] * inv, acc[3] * inv));
    }
    if (lane == 0 && lse != nullptr) lse[lrow] = total > 0.f ? M + logf(total) : -INFINITY;
}

}  // namespace attn
