// fa_fwd_kernel.cuh -- forward pass of exact attention for sm_100a.
//
// What it computes (FlashAttention-2 abstract; iplexlaw FlashAttention-2
// blog, "Tiling preserves the attention calculation"): for every query row i,
// O_i = sum_j softmax_j(scale * q_i.k_j) v_j over the visible keys, and the
// row's log-sum-exp.  K and V stream through shared memory in 128-row blocks
// while an online softmax keeps a running maximum m and sum l per row and
// rescales the partial output, so the N x N scores never leave the SM.
//
// How it maps onto B200:
//  * One CTA owns two 128-row query tiles of one (batch, head) and walks the
//    key blocks once for both, so each K/V block fetched from L2/HBM feeds two
//    tiles of MMAs (the pages' "split Q, share K/V" idea at CTA granularity).
//  * Warp roles: warps 0-3 and 4-7 are the softmax warpgroups of tile 0 and
//    tile 1 (one thread per query row, which is also its TMEM lane); warp 8
//    issues tcgen05.mma from one thread; warp 9 issues TMA loads.
//  * TMEM (512 columns): S/P of tile t at columns [128t, 128t+128), the O
//    accumulator of tile t at [256 + d t, 256 + d t + d).  P is written back
//    as bf16 over the first 64 columns of S and read by the PV MMA straight
//    from TMEM.
//  * K and V blocks share one ring of shared-memory slots (order K0, V0, K1,
//    V1, ...) guarded by full/empty mbarriers; TMA zero-fills rows past N.
//  * Fewer non-matmul operations (blog, "Three changes improve GPU
//    utilisation"): the scale is folded into one FFMA before exp2, O is
//    rescaled only when a row's maximum grows by more than 2^8 (the stale
//    maximum is exact for the final result because l and O share it), and
//    only the diagonal block and the ragged last block are masked; causal
//    blocks above the diagonal are never loaded.
#pragma once

#include "sm100_ptx.cuh"

namespace fa {

// QK8: Q and K are e4m3 (one byte per element) and S = Q K^T runs as a
// kind::f8f6f4 MMA at twice the bf16 rate; P and V stay bf16.
// BIAS: an additive bf16 score bias b_ij, one [128 x 128] tile per query
// tile and key block, brought in by TMA.
// PV8 (with QK8): V is e4m3 too and O += P V also runs as a kind::f8f6f4
// MMA: P is scaled by 2^PV8_P_SHIFT and rounded to e4m3 in the softmax
// (a fixed per-block scale that puts the block's weights in e4m3's normal
// range), the deferred-rescale threshold drops to 2 (log2 units) so that the
// scaled weights stay below e4m3's maximum 448, and O is normalised by the
// sum of the rounded weights the MMA used.
template <int D, bool QK8 = false, bool BIAS = false, bool PV8 = false>
struct FwdTraits {
    static_assert(D == 64 || D == 128, "head dim");
    static_assert(!QK8 || D == 128, "e4m3 scores need 128-byte rows (d = 128)");
    static_assert(!(QK8 && BIAS), "one variant at a time");
    static_assert(!PV8 || QK8, "8-bit P V comes with 8-bit scores");
    static constexpr int BM = 128;                  // query rows per tile
    static constexpr int BN = 128;                  // key rows per block
    static constexpr int TILES = 2;                 // query tiles per CTA
    static constexpr int CHUNKS = D / 64;           // 128-byte swizzle column chunks (bf16)
    static constexpr int CHUNK_BYTES = 128 * 128;   // 128 rows x 128 B
    static constexpr int TILE_BYTES = BM * D * 2;   // one 128-row bf16 tile
    static constexpr int QK_ELEM = QK8 ? 1 : 2;     // bytes per Q / K element
    static constexpr int QK_CHUNKS = D * QK_ELEM / 128;
    static constexpr int QK_CHUNK_COLS = 128 / QK_ELEM;  // elements per swizzle chunk row
    static constexpr int QK_TILE_BYTES = BM * D * QK_ELEM;
    static constexpr int S_KSTEPS = D * QK_ELEM / 32;    // 32-byte K steps of S = Q K^T
    static constexpr int V_ELEM = PV8 ? 1 : 2;            // bytes per V element
    static constexpr int V_CHUNKS = D * V_ELEM / 128;
    static constexpr int V_CHUNK_COLS = 128 / V_ELEM;
    static constexpr int V_TILE_BYTES = BN * D * V_ELEM;
    // K steps of O += P V (32 bytes of P per row each: 16 bf16 or 32 e4m3
    // keys) and the bytes of V each step advances by.
    static constexpr int PV_KSTEPS = BN * V_ELEM / 32;
    static constexpr int PV_KSTEP_BYTES = (32 / V_ELEM) * 128;
    static constexpr int PV8_P_SHIFT = 6;
    static constexpr int NSLOT = (D == 128) ? (BIAS ? 3 : 4) : 8;
    static constexpr int Q_OFF = 0;
    static constexpr int KV_OFF = Q_OFF + TILES * QK_TILE_BYTES;
    // O staging for the epilogue: in the tile's own Q buffer when that holds
    // a bf16 tile, else in a region of its own (an e4m3 Q tile is half size).
    static constexpr int OST_OFF = KV_OFF + NSLOT * TILE_BYTES;
    // Bias tiles (BIAS): one [128 rows][128 keys] bf16 tile per query tile,
    // two 64-key swizzle chunks each, single-buffered: the softmax reads its
    // row of the tile right after the scores, long before the next one.
    static constexpr int BIAS_TILE = BM * BN * 2;
    static constexpr int BIAS_OFF = OST_OFF + (QK8 ? TILES * TILE_BYTES : 0);
    static constexpr int BAR_OFF = BIAS_OFF + (BIAS ? TILES * BIAS_TILE : 0);
    // q, full[NSLOT], empty[NSLOT], s_full[2], p_ready[2], o_final[2],
    // mma_done, bias_full[2], bias_empty[2], p_half[2]
    static constexpr int NBAR = 1 + 2 * NSLOT + 2 + 2 + 2 + 1 + 4 + 2;
    static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
    static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;  // + alignment slack
    static constexpr int NUM_THREADS = 384;  // 3 warpgroups; warps 10-11 idle
    static constexpr int MMA_WARP = 8;
    static constexpr int LOAD_WARP = 9;
    static constexpr int BIAS_WARP = 10;
    // Register split: softmax warpgroups grow, the MMA/TMA warpgroup shrinks.
    // The causal softmax (diagonal masks) keeps 208; the non-causal MMA
    // thread needs 104 to hold its descriptors and addresses without
    // spilling.  Both splits total the same 64,512 registers.
    static __host__ __device__ constexpr uint32_t reg_softmax(bool causal) { return causal ? 208 : 200; }
    static __host__ __device__ constexpr uint32_t reg_control(bool causal) { return causal ? 88 : 104; }
    static constexpr int REG_BUDGET = 128 * (2 * 208 + 88);
    static_assert(2 * 200 + 104 == 2 * 208 + 88, "both splits use the same registers");
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t IDESC_S = QK8 ? idesc_e4m3_f32(128, BN) : idesc_bf16_f32(128, BN, 0, 0);
    static constexpr uint32_t IDESC_PV =
        PV8 ? idesc_e4m3_f32_bmn(128, D) : idesc_bf16_f32(128, D, 0, 1);
    // deferred-rescale threshold (log2 units)
    static constexpr float TAU = PV8 ? 2.0f : 8.0f;
    // The softmax signals P per 64-key half and the PV MMA starts on the
    // first half early.  At d = 64 (softmax-bound) that gains; at d = 128
    // the extra TMEM-store wait in the middle of the softmax costs more.
    static constexpr bool PSPLIT = (D == 64);
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct FwdParams {
    float* lse;            // [BH, N]
    unsigned int* err;     // device error word
    int N;
    int n_qpairs;          // ceil(N / 256)
    int bh_count;          // B * H
    float scale_log2;      // scale * log2(e)
    int H;                 // heads (to split b*H + h)
    int bias_batch;        // bias varies with the batch index (else shared)
    int bias_heads;        // bias varies with the head index (else shared)
    int strict;            // causal mask without the diagonal: key j visible iff j < i
    float o_scale;         // PV8: V's dequantisation factor (O = o_scale * P V / l)
};

// One softmax row over a 128-key block: p = exp2(s * scale*log2(e) - m) in
// pairs (f32x2 FFMA for the argument), packed to bf16 and written over the
// first 64 TMEM columns of S; adds the fp32 sum of p (for the LSE) to l and
// the sum of the bf16-rounded p (for normalising O) to lr.  The rounded
// weights are summed straight from the packed bf16 pairs with mixed-precision
// adds (exact widening, fp32 sum).  Every fourth pair's exponentials run on
// the FMA pipe (exp2_fma2) instead of the MUFU unit: one MUFU ex2 per score
// against 4*d tensor FLOP per score puts the two units at about the same time
// per block at d = 128 and MUFU at twice the tensor time at d = 64, so moving
// a quarter of the exponentials to the FMA pipe shortens the softmax that
// each tile's next MMAs wait for.  PSPLIT: the first 64 keys' P is made
// visible to the tensor core and `half_bar` arrived on before the second half
// is computed.
template <bool PSPLIT>
__device__ __forceinline__ void softmax_block_exp(const uint32_t (&sr)[4][32], float sl2,
                                                  float m, uint32_t s_tm, float& l, float& lr,
                                                  uint64_t* half_bar) {
    const uint64_t sl2x2 = f2_pack(sl2, sl2);
    const uint64_t negm2 = f2_pack(-m, -m);
    uint64_t sum2[2] = {0ull, 0ull};
    float rs[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            const int c = 64 * h + 2 * e;
            const uint64_t x2 = ffma2(f2_pack(__uint_as_float(sr[c >> 5][c & 31]),
                                              __uint_as_float(sr[(c + 1) >> 5][(c + 1) & 31])),
                                      sl2x2, negm2);
            float x0, x1;
            f2_unpack(x2, x0, x1);
            float p0, p1;
            if ((e & 3) == 3) {
                exp2_fma2(x0, x1, p0, p1);
            } else {
                p0 = ex2_approx(x0);
                p1 = ex2_approx(x1);
            }
            sum2[e & 1] = fadd2(sum2[e & 1], f2_pack(p0, p1));
            pk[e] = pack_bf16x2(p0, p1);
            add_bf16x2_to_f32(pk[e], rs[2 * (e & 1)], rs[2 * (e & 1) + 1]);
        }
        tmem_st32(s_tm + 32u * h, pk);
        if (PSPLIT && h == 0) {
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(half_bar);
        }
    }
    float a0, a1;
    f2_unpack(fadd2(sum2[0], sum2[1]), a0, a1);
    l += a0 + a1;
    lr += (rs[0] + rs[1]) + (rs[2] + rs[3]);
}

// The same for 8-bit P V (PV8): each weight is scaled by 2^shift (added to
// its exponent) and rounded to e4m3, four per TMEM column over the first 32
// columns of S; lr sums the rounded scaled weights (what the PV MMA uses), l
// the fp32 unscaled ones.
__device__ __forceinline__ void softmax_block_exp8(const uint32_t (&sr)[4][32], float sl2,
                                                   float m, uint32_t s_tm, float& l, float& lr,
                                                   int shift) {
    const uint64_t sl2x2 = f2_pack(sl2, sl2);
    // exp2(x - m + shift) = 2^shift * p: the scale rides in the exponent
    const uint64_t negm2 = f2_pack(static_cast<float>(shift) - m, static_cast<float>(shift) - m);
    uint64_t sum2[2] = {0ull, 0ull};
    float rs[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            const int c = 64 * h + 2 * e;
            const uint64_t x2 = ffma2(f2_pack(__uint_as_float(sr[c >> 5][c & 31]),
                                              __uint_as_float(sr[(c + 1) >> 5][(c + 1) & 31])),
                                      sl2x2, negm2);
            float x0, x1;
            f2_unpack(x2, x0, x1);
            float p0, p1;
            if ((e & 3) == 3) {
                exp2_fma2(x0, x1, p0, p1);
            } else {
                p0 = ex2_approx(x0);
                p1 = ex2_approx(x1);
            }
            sum2[e & 1] = fadd2(sum2[e & 1], f2_pack(p0, p1));
            const uint16_t q = pack_e4m3x2(p0, p1);
            add_e4m3x2_to_f32(q, rs[2 * (e & 1)], rs[2 * (e & 1) + 1]);
            if (e & 1)
                pk[e >> 1] |= static_cast<uint32_t>(q) << 16;
            else
                pk[e >> 1] = q;
        }
        tmem_st16(s_tm + 16u * h, pk);
    }
    float a0, a1;
    f2_unpack(fadd2(sum2[0], sum2[1]), a0, a1);
    l += (a0 + a1) * exp2f(static_cast<float>(-shift));
    lr += (rs[0] + rs[1]) + (rs[2] + rs[3]);
}

template <int D, bool CAUSAL, bool QK8 = false, bool BIAS = false, bool PV8 = false>
__global__ void __launch_bounds__(384, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                  const __grid_constant__ CUtensorMap tmB, const FwdParams p) {
    using T = FwdTraits<D, QK8, BIAS, PV8>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::BAR_OFF);
    uint64_t* bar_q = bars;
    uint64_t* full = bars + 1;
    uint64_t* empty = full + T::NSLOT;
    uint64_t* s_full = empty + T::NSLOT;
    uint64_t* p_ready = s_full + 2;
    uint64_t* o_final = p_ready + 2;
    uint64_t* mma_done = o_final + 2;
    uint64_t* bias_full = mma_done + 1;
    uint64_t* bias_empty = bias_full + 2;
    uint64_t* p_half = bias_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + T::MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + T::MISC_OFF + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // Non-causal: consecutive CTAs share a head (K/V reuse in L2).  Causal:
    // heavy tiles first -- the last query pair of every head has the most key
    // blocks, so the grid walks query pairs from the end.
    int qp, bh;
    if (CAUSAL) {
        bh = static_cast<int>(blockIdx.x % p.bh_count);
        qp = p.n_qpairs - 1 - static_cast<int>(blockIdx.x / p.bh_count);
    } else {
        qp = static_cast<int>(blockIdx.x % p.n_qpairs);
        bh = static_cast<int>(blockIdx.x / p.n_qpairs);
    }
    const int N = p.N;
    const int q0 = qp * 256;
    const int n_kv = (N + T::BN - 1) / T::BN;
    const int n0 = CAUSAL ? min(n_kv, 2 * qp + 1) : n_kv;  // key blocks of tile 0
    const int n1 = CAUSAL ? min(n_kv, 2 * qp + 2) : n_kv;  // key blocks of tile 1
    // Causal: the key blocks are walked from the diagonal down, so tile 1's
    // extra block (its diagonal, hidden from tile 0) comes first, while tile
    // 0's first scores are computed, and both tiles end on block 0 together
    // (in ascending order tile 1's last block would run with no partner).
    // Iteration i visits key block kv_block(i); tile 0 joins at i = off0.
    const int off0 = CAUSAL ? n1 - n0 : 0;
    auto kv_block = [&](int i) { return CAUSAL ? n1 - 1 - i : i; };

    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        for (int s = 0; s < T::NSLOT; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(&s_full[t], 1);
            mbar_init(&p_ready[t], 128);
            mbar_init(&o_final[t], 1);
            mbar_init(&bias_full[t], 1);
            mbar_init(&bias_empty[t], 128);
            mbar_init(&p_half[t], 128);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
        // Q and the first key/value block are requested here, so that their
        // latency overlaps the TMEM allocation and the block-wide sync; the
        // producer warp continues with the second block.
        mbar_arrive_expect_tx(bar_q, T::TILES * T::QK_TILE_BYTES);
        for (int t = 0; t < T::TILES; ++t)
            for (int c = 0; c < T::QK_CHUNKS; ++c)
                tma_load_3d(smem + T::Q_OFF + t * T::QK_TILE_BYTES + c * T::CHUNK_BYTES, &tmQ,
                            bar_q, c * T::QK_CHUNK_COLS, q0 + 128 * t, bh);
        for (int h = 0; h < 2; ++h) {  // slots 0 and 1: K and V of iteration 0
            mbar_arrive_expect_tx(&full[h], h ? T::V_TILE_BYTES : T::QK_TILE_BYTES);
            uint8_t* dst = smem + T::KV_OFF + h * T::TILE_BYTES;
            const int nch = h ? T::V_CHUNKS : T::QK_CHUNKS;
            const int ccols = h ? T::V_CHUNK_COLS : T::QK_CHUNK_COLS;
            for (int c = 0; c < nch; ++c)
                tma_load_3d(dst + c * T::CHUNK_BYTES, h ? &tmV : &tmK, &full[h], c * ccols,
                            kv_block(0) * T::BN, bh);
        }
    }
    if (warp == T::MMA_WARP) {
        tmem_alloc(tmem_slot, T::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == T::LOAD_WARP && lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        tma_prefetch_desc(&tmO);
        if (BIAS) tma_prefetch_desc(&tmB);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const AbortState st{abort_flag, p.err};
    if (warp >= 8) {
      setmaxnreg_dec<T::reg_control(CAUSAL)>();
      if (warp == T::LOAD_WARP) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            bool ok = true;
            int issued = 2;  // Q and iteration 0's K, V were issued at set-up
            for (int j = 1; j < n1 && ok; ++j) {
                for (int h = 0; h < 2; ++h) {  // 0: K_j, 1: V_j
                    const int idx = 2 * j + h;
                    const int slot = idx % T::NSLOT;
                    const uint32_t par = (idx / T::NSLOT) & 1;
                    if (!mbar_wait(&empty[slot], par ^ 1u, st)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[slot], h ? T::V_TILE_BYTES : T::QK_TILE_BYTES);
                    uint8_t* dst = smem + T::KV_OFF + slot * T::TILE_BYTES;
                    const int nch = h ? T::V_CHUNKS : T::QK_CHUNKS;
                    const int ccols = h ? T::V_CHUNK_COLS : T::QK_CHUNK_COLS;
                    for (int c = 0; c < nch; ++c)
                        tma_load_3d(dst + c * T::CHUNK_BYTES, h ? &tmV : &tmK, &full[slot],
                                    c * ccols, kv_block(j) * T::BN, bh);
                    ++issued;
                }
            }
            if (!ok) {
                // Let copies still in flight land before the CTA exits.
                for (int idx = max(0, issued - T::NSLOT); idx < issued; ++idx)
                    mbar_wait_bounded(&full[idx % T::NSLOT], (idx / T::NSLOT) & 1);
                mbar_wait_bounded(bar_q, 0);
            }
        }
        __syncwarp();
      } else if (BIAS && warp == T::BIAS_WARP) {
        // ------------------------------------------------ bias tile producer
        if (lane == 0) {
            const int b = bh / p.H, h = bh % p.H;
            const int bz = (p.bias_batch ? b : 0) * (p.bias_heads ? p.H : 1) +
                           (p.bias_heads ? h : 0);
            int issued[2] = {0, 0};
            bool ok = true;
            for (int j = 0; j < n1 && ok; ++j) {
                for (int t = 0; t < 2; ++t) {
                    if (t == 0 && (j < off0 || j - off0 >= n0)) continue;
                    // the previous tile of this query tile must have been read
                    if (issued[t] > 0 &&
                        !mbar_wait(&bias_empty[t], (issued[t] - 1) & 1, st)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bias_full[t], T::BIAS_TILE);
                    uint8_t* dst = smem + T::BIAS_OFF + t * T::BIAS_TILE;
                    for (int c = 0; c < 2; ++c)
                        tma_load_3d(dst + c * T::CHUNK_BYTES, &tmB, &bias_full[t],
                                    kv_block(j) * T::BN + 64 * c, q0 + 128 * t, bz);
                    ++issued[t];
                }
            }
            if (!ok)  // let the copies in flight land before the CTA exits
                for (int t = 0; t < 2; ++t)
                    if (issued[t]) mbar_wait_bounded(&bias_full[t], (issued[t] - 1) & 1);
        }
        __syncwarp();
      } else if (warp == T::MMA_WARP) {
        // ------------------------------------------------ MMA issuer
        // This one thread's instruction stream paces the kernel: it shares
        // its SM sub-partition with two busy softmax warps, and a probe that
        // added 32 dependent integer instructions per key block cost 8-12%
        // of the forward's rate.  So what does not change from block to
        // block is computed once (operand descriptors, barrier addresses)
        // and the ring position advances by adds.
        if (lane == 0) {
            const uint32_t q_base = smem_u32(smem + T::Q_OFF);
            const uint32_t kv_base = smem_u32(smem + T::KV_OFF);
            const uint64_t dq[2] = {sdesc_sw128(q_base, 16, 1024),
                                    sdesc_sw128(q_base + T::QK_TILE_BYTES, 16, 1024)};
            const uint64_t dk_base = sdesc_sw128(kv_base, 16, 1024);             // K in slot 0
            const uint64_t dv_base = sdesc_sw128(kv_base, T::CHUNK_BYTES, 1024);  // V in slot 0
            // Barrier addresses: one register (the barrier block's base) plus
            // compile-time offsets, so this thread's register budget stays small.
            const uint32_t bar_a = smem_u32(bars);
            constexpr uint32_t FULL = 8u * 1, EMPTY = FULL + 8u * T::NSLOT, SFULL = EMPTY + 8u * T::NSLOT;
            constexpr uint32_t PREADY = SFULL + 16u, OFINAL = PREADY + 16u;
            constexpr uint32_t PHALF = OFINAL + 16u + 8u + 32u;  // after mma_done, bias_full/empty
            const uint32_t full_a = bar_a + FULL, empty_a = bar_a + EMPTY, sfull_a = bar_a + SFULL;
            const uint32_t pready_a = bar_a + PREADY, phalf_a = bar_a + PHALF, ofinal_a = bar_a + OFINAL;
            // S_t = Q_t K^T : M=128, N=128, K=D, both operands K-major;
            // each MMA consumes 32 bytes of every row (16 bf16 or 32 e4m3).
            // dk: the descriptor of the K slot; K steps add byte offsets.
            auto mma_s = [&](int t, uint64_t dk) {
#pragma unroll
                for (int k = 0; k < T::S_KSTEPS; ++k) {
                    const uint32_t off = (k >> 2) * T::CHUNK_BYTES + (k & 3) * 32;
                    const uint64_t a = sdesc_add(dq[t], off);
                    const uint64_t b = sdesc_add(dk, off);
                    if constexpr (QK8)
                        umma_ss_f8(tmem + 128u * t, a, b, T::IDESC_S, k > 0 ? 1u : 0u);
                    else if (k == 0)
                        umma_ss_c<false>(tmem + 128u * t, a, b, T::IDESC_S);
                    else
                        umma_ss_c<true>(tmem + 128u * t, a, b, T::IDESC_S);
                }
            };
            // O_t += P_t V : M=128, N=D, K=128; P from TMEM, V MN-major.
            // K steps [k0, k1) of O_t += P_t V (16 keys each); dv: the V slot.
            auto mma_pv = [&](int t, uint64_t dv, bool accumulate, int k0, int k1) {
#pragma unroll
                for (int k = k0; k < k1; ++k) {
                    const uint32_t a = tmem + 128u * t + 8u * k;  // 32 bytes of P per row
                    const uint64_t b = sdesc_add(dv, k * T::PV_KSTEP_BYTES);
                    const uint32_t acc = (k > 0 || accumulate) ? 1u : 0u;
                    if constexpr (PV8)
                        umma_ts_f8(tmem + 256u + D * t, a, b, T::IDESC_PV, acc);
                    else if (k == 0)
                        umma_ts(tmem + 256u + D * t, a, b, T::IDESC_PV, acc);
                    else
                        umma_ts_c<true>(tmem + 256u + D * t, a, b, T::IDESC_PV);
                }
            };
            // PV of tile t for the block whose P has phase `par`: in two
            // 64-key halves when the softmax signals them separately.
            auto pv_tile = [&](int t, uint64_t dv, bool acc, uint32_t par) -> bool {
                if constexpr (T::PSPLIT) {
                    if (!mbar_wait_s(phalf_a + 8u * t, par, st)) return false;
                    tc_fence_after();
                    mma_pv(t, dv, acc, 0, T::PV_KSTEPS / 2);
                    if (!mbar_wait_s(pready_a + 8u * t, par, st)) return false;
                    tc_fence_after();
                    mma_pv(t, dv, true, T::PV_KSTEPS / 2, T::PV_KSTEPS);
                } else {
                    if (!mbar_wait_s(pready_a + 8u * t, par, st)) return false;
                    tc_fence_after();
                    mma_pv(t, dv, acc, 0, T::PV_KSTEPS);
                }
                return true;
            };
            // Tile 0 takes part in iterations [off0, n1) (off0 + n0 = n1);
            // its own block count (for its barrier phases) is i - off0.
            auto act0 = [&](int i) { return i >= off0; };
            bool ok = mbar_wait(bar_q, 0, st) && mbar_wait_s(full_a, 0, st);
            if (ok) {
                tc_fence_after();
                if (act0(0)) {
                    mma_s(0, dk_base);
                    umma_commit_s(sfull_a);
                }
                mma_s(1, dk_base);
                umma_commit_s(sfull_a + 8u);
                umma_commit_s(empty_a);
            }
            // Ring slot and phase parity of K_j (position 2j); V_{j-1} sits
            // one position before it.
            uint32_t ks = 2u % T::NSLOT, kp = (2u / T::NSLOT) & 1u;
            for (int j = 1; j < n1 && ok; ++j) {
                const uint32_t vs = ks ? ks - 1u : T::NSLOT - 1u;
                const uint32_t vp = ks ? kp : kp ^ 1u;
                ok = mbar_wait_s(full_a + 8u * ks, kp, st) && mbar_wait_s(full_a + 8u * vs, vp, st);
                if (!ok) break;
                tc_fence_after();
                const uint64_t dk = sdesc_add(dk_base, ks * T::TILE_BYTES);
                const uint64_t dv = sdesc_add(dv_base, vs * T::TILE_BYTES);
                if (act0(j - 1)) {
                    const int l0 = j - 1 - off0;  // never tile 0's last block (that is j = n1)
                    if (!(ok = pv_tile(0, dv, l0 > 0, l0 & 1))) break;
                }
                if (act0(j)) {
                    mma_s(0, dk);
                    umma_commit_s(sfull_a);
                }
                if (!(ok = pv_tile(1, dv, j - 1 > 0, (j - 1) & 1))) break;
                umma_commit_s(empty_a + 8u * vs);
                mma_s(1, dk);
                umma_commit_s(sfull_a + 8u);
                umma_commit_s(empty_a + 8u * ks);
                ks += 2u;
                if (ks >= T::NSLOT) {
                    ks -= T::NSLOT;
                    kp ^= 1u;
                }
            }
            if (ok) {  // V of the last block, one position before K_{n1}'s
                const int jl = n1 - 1;
                const uint32_t vs = ks ? ks - 1u : T::NSLOT - 1u;
                const uint32_t vp = ks ? kp : kp ^ 1u;
                const uint64_t dv = sdesc_add(dv_base, vs * T::TILE_BYTES);
                ok = mbar_wait_s(full_a + 8u * vs, vp, st);
                if (ok && act0(jl)) {
                    tc_fence_after();
                    const int l0 = jl - off0;
                    ok = pv_tile(0, dv, l0 > 0, l0 & 1);
                    if (ok) umma_commit_s(ofinal_a);
                }
                if (ok) {
                    tc_fence_after();
                    ok = pv_tile(1, dv, jl > 0, jl & 1);
                }
                if (ok) {
                    umma_commit_s(ofinal_a + 8u);
                    umma_commit_s(empty_a + 8u * vs);
                }
            }
            // No MMA may still be running when TMEM is released.
            umma_commit(mma_done);
            mbar_wait_bounded(mma_done, 0);
        }
        __syncwarp();
      }
    } else {
        // ------------------------------------------------ softmax warpgroups
        setmaxnreg_inc<T::reg_softmax(CAUSAL)>();
        const int t = warp >> 2;         // query tile
        const int lg = warp & 3;         // TMEM lane group of this warp
        const int r = lg * 32 + lane;    // row within the tile = TMEM lane
        const int row0 = q0 + 128 * t;
        const int row = row0 + r;
        const int nt = t ? n1 : n0;
        const uint32_t lane_off = static_cast<uint32_t>(lg * 32) << 16;
        const uint32_t s_tm = tmem + lane_off + 128u * t;
        const uint32_t o_tm = tmem + lane_off + 256u + D * t;
        const float sl2 = p.scale_log2;
        float m = -INFINITY;  // reference maximum, log2 units of scaled scores
        float l = 0.f;        // running sum of exp2(score - m), fp32 (for LSE)
        float lr = 0.f;       // the same sum over the bf16-rounded weights the
                              // PV MMA uses (normalises O consistently)
        bool ok = true;

        for (int j = 0; j < nt; ++j) {
            ok = __all_sync(0xffffffffu, mbar_wait(&s_full[t], j & 1, st));
            if (!ok) break;
            tc_fence_after();
            uint32_t sr[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(s_tm + 32u * c, sr[c]);
            tmem_ld_wait();
            if constexpr (BIAS) {
                // Scores become t = s * scale*log2(e) + b * log2(e), the
                // exponent in base 2 (so the rest runs with unit scale).
                ok = __all_sync(0xffffffffu, mbar_wait(&bias_full[t], j & 1, st));
                if (!ok) break;
                const uint8_t* brow = smem + T::BIAS_OFF + t * T::BIAS_TILE + r * 128;
                const uint64_t sl2x2 = f2_pack(sl2, sl2);
                const uint64_t lg2x2 = f2_pack(1.4426950408889634f, 1.4426950408889634f);
#pragma unroll
                for (int u = 0; u < 16; ++u) {  // keys 8u .. 8u+7
                    const uint4 bv = *reinterpret_cast<const uint4*>(
                        brow + (u >> 3) * T::CHUNK_BYTES + (((u & 7) ^ (r & 7)) << 4));
                    const uint32_t w[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int c = 8 * u + 2 * i;
                        const uint64_t b2 = f2_pack(__uint_as_float(w[i] << 16),
                                                    __uint_as_float(w[i] & 0xffff0000u));
                        const uint64_t s2 = f2_pack(__uint_as_float(sr[c >> 5][c & 31]),
                                                    __uint_as_float(sr[c >> 5][(c & 31) + 1]));
                        float t0, t1;
                        f2_unpack(ffma2(s2, sl2x2, ffma2(b2, lg2x2, 0ull)), t0, t1);
                        sr[c >> 5][c & 31] = __float_as_uint(t0);
                        sr[c >> 5][(c & 31) + 1] = __float_as_uint(t1);
                    }
                }
                mbar_arrive(&bias_empty[t]);
            }
            constexpr float kUnit = 1.0f;
            const float sl2e = BIAS ? kUnit : sl2;  // scale still to apply to sr

            // tile t's j-th block: key block nt-1-j when walking down
            const int kv0 = (CAUSAL ? nt - 1 - j : j) * T::BN;
            // Only the ragged last block and (causal) the diagonal block hold
            // hidden scores; the test is uniform over the tile.
            const bool masked_block =
                (kv0 + T::BN > N) || (CAUSAL && kv0 + T::BN - 1 > row0);
            if (masked_block) {
                int lim = min(T::BN, N - kv0);
                if (CAUSAL) lim = min(lim, row - kv0 + 1 - p.strict);
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    if (c >= lim) sr[c >> 5][c & 31] = __float_as_uint(-INFINITY);
            }
            // Row maximum: eight independent chains, then a tree.
            float mx[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) mx[i] = __uint_as_float(sr[0][i]);
#pragma unroll
            for (int c = 8; c < 128; c += 8)
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    mx[i] = fmaxf(mx[i], __uint_as_float(sr[(c + i) >> 5][(c + i) & 31]));
            mx[0] = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                          fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
            const float m_blk = mx[0] * sl2e;
            const float m_new = (m_blk > m + T::TAU) ? m_blk : m;
            if (j > 0) {
                const bool grow = m_new != m;
                if (__any_sync(0xffffffffu, grow)) {
                    const float alpha = grow ? ex2_approx(m - m_new) : 1.0f;
                    l *= alpha;
                    lr *= alpha;
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t o[32];
                        tmem_ld32(o_tm + 32u * c, o);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tmem_st32(o_tm + 32u * c, o);
                    }
                }
            }
            m = m_new;
            // A row that has seen no visible key yet (only the strict causal
            // mask's row 0) keeps m = -inf; its weights are exp2(-inf) = 0.
            if constexpr (PV8)
                softmax_block_exp8(sr, sl2e, m == -INFINITY ? 0.f : m, s_tm, l, lr,
                                   T::PV8_P_SHIFT);
            else
                softmax_block_exp<T::PSPLIT>(sr, sl2e, m == -INFINITY ? 0.f : m, s_tm, l, lr,
                                             &p_half[t]);
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&p_ready[t]);
        }

        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&o_final[t], 0, st));
        if (ok) {
            tc_fence_after();
            // A row with no visible key (strict causal row 0) keeps m = -inf:
            // O = 0, LSE = -inf.  (Its weights are not all 0 -- the FMA-pipe
            // exp2 returns 2^-126 for -inf -- so lr alone cannot tell.)
            const float inv_l = m == -INFINITY ? 0.f : (PV8 ? p.o_scale : 1.0f) / lr;
            const float lse_val = (m + log2f(l)) * 0.6931471805599453f;
            // Stage O (bf16, 128-byte swizzle) in this tile's Q buffer, which
            // no MMA reads any more (e4m3 scores: in the staging region),
            // then store this warp's 32 rows by TMA.
            uint8_t* stage = smem + (QK8 ? T::OST_OFF : T::Q_OFF) + t * T::TILE_BYTES +
                             lg * 32 * 128;
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(o_tm + 32u * c, o);
                tmem_ld_wait();
                uint8_t* chunk = stage + (c >> 1) * T::CHUNK_BYTES;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    uint4 v;
                    v.x = pack_bf16x2(__uint_as_float(o[8 * u + 0]) * inv_l,
                                      __uint_as_float(o[8 * u + 1]) * inv_l);
                    v.y = pack_bf16x2(__uint_as_float(o[8 * u + 2]) * inv_l,
                                      __uint_as_float(o[8 * u + 3]) * inv_l);
                    v.z = pack_bf16x2(__uint_as_float(o[8 * u + 4]) * inv_l,
                                      __uint_as_float(o[8 * u + 5]) * inv_l);
                    v.w = pack_bf16x2(__uint_as_float(o[8 * u + 6]) * inv_l,
                                      __uint_as_float(o[8 * u + 7]) * inv_l);
                    *reinterpret_cast<uint4*>(chunk + sw128_offset(lane, (c & 1) * 4 + u)) = v;
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            const int wrow0 = row0 + lg * 32;
            if (lane == 0 && wrow0 < N) {
                for (int c = 0; c < T::CHUNKS; ++c)
                    tma_store_3d(&tmO, stage + c * T::CHUNK_BYTES, c * 64, wrow0, bh);
                bulk_commit_group();
                bulk_wait_group_read0();
            }
            if (row < N) p.lse[static_cast<size_t>(bh) * N + row] = lse_val;
        }
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == T::MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem, T::TMEM_COLS);
    }
}

}  // namespace fa
