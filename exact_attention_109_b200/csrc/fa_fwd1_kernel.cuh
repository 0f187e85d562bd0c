// fa_fwd1_kernel.cuh -- the forward pass with one 128-row query tile at a
// time per CTA, two CTAs per SM, persistent over tiles, for short sequences.
//
// Same arithmetic as fa_fwd_kernel (FlashAttention-2 abstract; iplexlaw blog,
// "Tiling preserves the attention calculation": per query row an online
// softmax over 128-key blocks, the partial output rescaled when the running
// maximum grows) and the same softmax code, but a CTA works on a single query
// tile at a time and needs only 256 TMEM columns (S/P at [0, 128), O at
// [128, 128 + d)) and about 112 KB of shared memory, so two CTAs share an SM.
// When a sequence is short a tile has only a few key blocks, and the fixed
// cost around each tile -- barrier and TMEM set-up, the first TMA round trip,
// the epilogue, the gap before the next CTA starts -- is as long as its work
// (the blog's "Three changes improve GPU utilisation": keep the units busy at
// every sequence length).  So each CTA walks tiles tile0, tile0 + grid, ...
// (causal: the longest tiles first) and hides that cost: set-up happens once;
// the next tile's Q is requested as soon as the current tile's last score
// MMA has completed and its K/V blocks stream through the same ring; its
// first score MMA runs while the softmax warps write out the current tile's
// O (which they hand back with an mbarrier before the next PV overwrites it);
// and the second CTA on the SM fills the remaining gaps.  The price is one
// S buffer per CTA: the score MMA of key block j+1 waits until the softmax of
// block j has written P.
//
// Roles (256 threads = 2 warpgroups): warps 0-3 the softmax (one thread per
// query row = TMEM lane), warp 4 issues tcgen05.mma, warp 5 issues TMA, warps
// 6-7 idle.  K and V alternate through a ring of slots (the CTA's running
// count of K/V tiles picks the slot) under full/empty mbarriers; every wait is
// bounded.
#pragma once

#include "fa_fwd_kernel.cuh"

namespace fa {

template <int D>
struct Fwd1Traits {
    static_assert(D == 64 || D == 128, "head dim");
    static constexpr int BM = 128;
    static constexpr int BN = 128;
    static constexpr int CHUNKS = D / 64;
    static constexpr int CHUNK_BYTES = 128 * 128;
    static constexpr int TILE_BYTES = BM * D * 2;
    static constexpr int NSLOT = (D == 128) ? 2 : 4;
    static constexpr int Q_OFF = 0;
    static constexpr int KV_OFF = Q_OFF + TILE_BYTES;
    static constexpr int OST_OFF = KV_OFF + NSLOT * TILE_BYTES;  // O staging
    static constexpr int OST_WARP = 32 * 128;  // bf16 [32 rows][64 columns] per warp
    static constexpr int BAR_OFF = OST_OFF + 4 * OST_WARP;
    // q_full, q_empty, full[NSLOT], empty[NSLOT], s_full, p_ready, p_half,
    // o_final, o_free, mma_done
    static constexpr int NBAR = 2 + 2 * NSLOT + 6;
    static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
    // No alignment slack: the kernel checks that the dynamic shared memory
    // starts on a 1024-byte boundary and reports kErrLayout if not.
    static constexpr int SMEM_BYTES = MISC_OFF + 16;
    static constexpr int NUM_THREADS = 256;
    static constexpr int MMA_WARP = 4;
    static constexpr int LOAD_WARP = 5;
    static constexpr uint32_t REG_SOFTMAX = 184;
    static constexpr uint32_t REG_CONTROL = 72;
    static constexpr int REG_BUDGET = 128 * (REG_SOFTMAX + REG_CONTROL);
    static constexpr uint32_t TMEM_COLS = 256;
    static constexpr uint32_t O_COL = 128;
    static constexpr uint32_t IDESC_S = idesc_bf16_f32(128, BN, 0, 0);
    static constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, 0, 1);
    static constexpr float TAU = 8.0f;
    static constexpr bool PSPLIT = (D == 64);
    // two CTAs per SM, each with the 1 KB the system reserves per block
    static_assert(2 * (SMEM_BYTES + 1024) <= 233472, "two CTAs per SM");
};

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(256, 2)
    fa_fwd1_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                   const FwdParams p) {
    using T = Fwd1Traits<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw;
    if (smem_u32(smem) & 1023u) {  // the same for every thread of the block
        if (threadIdx.x == 0) atomicOr(p.err, kErrLayout);
        return;
    }

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::BAR_OFF);
    uint64_t* q_full = bars;
    uint64_t* q_empty = bars + 1;
    uint64_t* full = bars + 2;
    uint64_t* empty = full + T::NSLOT;
    uint64_t* s_full = empty + T::NSLOT;
    uint64_t* p_ready = s_full + 1;
    uint64_t* p_half = p_ready + 1;
    uint64_t* o_final = p_half + 1;
    uint64_t* o_free = o_final + 1;
    uint64_t* mma_done = o_free + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + T::MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + T::MISC_OFF + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int N = p.N;
    const int n_qt = (N + T::BM - 1) / T::BM;
    const int n_kv = (N + T::BN - 1) / T::BN;
    const int items = p.bh_count * n_qt;
    // Tile `it` = query tile qt of head bh.  Causal: the last tiles of every
    // head (most key blocks) first; non-causal: a head's tiles adjacent (K/V
    // reuse in L2).  Each CTA takes every gridDim.x-th tile.
    auto decode = [&](int it, int& qt, int& bh) {
        if (CAUSAL) {
            bh = it % p.bh_count;
            qt = n_qt - 1 - it / p.bh_count;
        } else {
            qt = it % n_qt;
            bh = it / n_qt;
        }
    };
    auto n_blocks = [&](int qt) { return CAUSAL ? min(n_kv, qt + 1) : n_kv; };
    // causal: from the diagonal down, so the masked block comes first
    auto kv_block = [&](int n, int i) { return CAUSAL ? n - 1 - i : i; };

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int s = 0; s < T::NSLOT; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(s_full, 1);
        mbar_init(p_ready, 128);
        mbar_init(p_half, 128);
        mbar_init(o_final, 1);
        mbar_init(o_free, 128);
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
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
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const AbortState st{abort_flag, p.err};
    if (warp >= 4) {
      setmaxnreg_dec<T::REG_CONTROL>();
      if (warp == T::LOAD_WARP) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            bool ok = true;
            int idx = 0;  // K/V tiles requested so far
            int nq = 0;   // Q tiles requested so far
            for (int it = blockIdx.x; it < items && ok; it += gridDim.x) {
                int qt, bh;
                decode(it, qt, bh);
                const int n = n_blocks(qt);
                // the previous tile's last score MMA has read Q
                if (nq > 0 && !(ok = mbar_wait(q_empty, (nq - 1) & 1, st))) break;
                mbar_arrive_expect_tx(q_full, T::TILE_BYTES);
                for (int c = 0; c < T::CHUNKS; ++c)
                    tma_load_3d(smem + T::Q_OFF + c * T::CHUNK_BYTES, &tmQ, q_full, c * 64,
                                qt * T::BM, bh);
                ++nq;
                for (int j = 0; j < n && ok; ++j) {
                    for (int h = 0; h < 2; ++h) {  // 0: K_j, 1: V_j
                        const int slot = idx % T::NSLOT;
                        if (!(ok = mbar_wait(&empty[slot], ((idx / T::NSLOT) & 1) ^ 1u, st)))
                            break;
                        mbar_arrive_expect_tx(&full[slot], T::TILE_BYTES);
                        for (int c = 0; c < T::CHUNKS; ++c)
                            tma_load_3d(smem + T::KV_OFF + slot * T::TILE_BYTES +
                                            c * T::CHUNK_BYTES,
                                        h ? &tmV : &tmK, &full[slot], c * 64,
                                        kv_block(n, j) * T::BN, bh);
                        ++idx;
                    }
                }
            }
            if (!ok) {  // let the copies already requested land before exiting
                for (int x = max(0, idx - T::NSLOT); x < idx; ++x)
                    mbar_wait_bounded(&full[x % T::NSLOT], (x / T::NSLOT) & 1);
                if (nq > 0) mbar_wait_bounded(q_full, (nq - 1) & 1);
            }
        }
        __syncwarp();
      } else if (warp == T::MMA_WARP) {
        // ------------------------------------------------ MMA issuer
        // This thread's instruction stream is on the kernel's critical path:
        // descriptors and barrier addresses are built once, and the ring
        // position is an unsigned counter (a mask and a shift per use).
        if (lane == 0) {
            const uint32_t q_base = smem_u32(smem + T::Q_OFF);
            const uint32_t kv_base = smem_u32(smem + T::KV_OFF);
            const uint64_t dq0 = sdesc_sw128(q_base, 16, 1024);
            const uint64_t dk_base = sdesc_sw128(kv_base, 16, 1024);             // K in slot 0
            const uint64_t dv_base = sdesc_sw128(kv_base, T::CHUNK_BYTES, 1024);  // V in slot 0
            const uint32_t qfull_a = smem_u32(q_full), qempty_a = smem_u32(q_empty);
            const uint32_t full_a = smem_u32(full), empty_a = smem_u32(empty);
            const uint32_t sfull_a = smem_u32(s_full), pready_a = smem_u32(p_ready);
            const uint32_t phalf_a = smem_u32(p_half), ofinal_a = smem_u32(o_final);
            const uint32_t ofree_a = smem_u32(o_free);
            auto slot = [](uint32_t idx) { return idx % static_cast<uint32_t>(T::NSLOT); };
            auto slot_par = [](uint32_t idx) { return (idx / static_cast<uint32_t>(T::NSLOT)) & 1u; };
            // S = Q K^T: M=128, N=128, K=D, both K-major; dk: the K slot.
            auto mma_s = [&](uint64_t dk0) {
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint32_t off = (k >> 2) * T::CHUNK_BYTES + (k & 3) * 32;
                    if (k == 0)
                        umma_ss_c<false>(tmem, dq0, dk0, T::IDESC_S);
                    else
                        umma_ss_c<true>(tmem, sdesc_add(dq0, off), sdesc_add(dk0, off), T::IDESC_S);
                }
            };
            // O += P V: M=128, N=D, K=128 keys; P from TMEM, V MN-major.
            auto mma_pv = [&](uint64_t dv0, bool accumulate, int k0, int k1) {
#pragma unroll
                for (int k = k0; k < k1; ++k) {
                    if (k == 0)
                        umma_ts(tmem + T::O_COL, tmem, dv0, T::IDESC_PV, accumulate ? 1u : 0u);
                    else
                        umma_ts_c<true>(tmem + T::O_COL, tmem + 8u * k, sdesc_add(dv0, k * 2048),
                                        T::IDESC_PV);
                }
            };
            auto kdesc = [&](uint32_t idx) { return sdesc_add(dk_base, slot(idx) * T::TILE_BYTES); };
            auto vdesc = [&](uint32_t idx) { return sdesc_add(dv_base, slot(idx) * T::TILE_BYTES); };
            bool ok = true;
            uint32_t idx = 0;  // K/V tiles consumed so far
            uint32_t jb = 0;   // key blocks done so far (s_full / p_ready phases)
            uint32_t ni = 0;   // tiles done so far (q_full / o_final / o_free phases)
            for (int it = blockIdx.x; it < items && ok; it += gridDim.x) {
                int qt, bh;
                decode(it, qt, bh);
                const int n = n_blocks(qt);
                // S of the tile's first block overwrites the previous tile's
                // last P only after the PV that read it (MMAs from one thread
                // run in order).
                if (!(ok = mbar_wait_s(qfull_a, ni & 1u, st) &&
                           mbar_wait_s(full_a + 8u * slot(idx), slot_par(idx), st)))
                    break;
                tc_fence_after();
                mma_s(kdesc(idx));
                umma_commit_s(sfull_a);
                umma_commit_s(empty_a + 8u * slot(idx));
                ++idx;
                if (n == 1) umma_commit_s(qempty_a);
                for (int i = 0; i < n && ok; ++i, ++jb) {
                    const uint32_t iv = idx;  // V of block i
                    const uint32_t par = jb & 1u;
                    if (!(ok = mbar_wait_s(full_a + 8u * slot(iv), slot_par(iv), st))) break;
                    // the first PV of a tile overwrites O: the softmax warps
                    // must have read the previous tile's O out of TMEM
                    if (i == 0 && ni > 0 && !(ok = mbar_wait_s(ofree_a, (ni - 1) & 1u, st))) break;
                    const uint64_t dv = vdesc(iv);
                    if constexpr (T::PSPLIT) {
                        if (!(ok = mbar_wait_s(phalf_a, par, st))) break;
                        tc_fence_after();
                        mma_pv(dv, i > 0, 0, T::BN / 32);
                        if (!(ok = mbar_wait_s(pready_a, par, st))) break;
                        tc_fence_after();
                        mma_pv(dv, true, T::BN / 32, T::BN / 16);
                    } else {
                        if (!(ok = mbar_wait_s(pready_a, par, st))) break;
                        tc_fence_after();
                        mma_pv(dv, i > 0, 0, T::BN / 16);
                    }
                    umma_commit_s(empty_a + 8u * slot(iv));
                    ++idx;
                    if (i + 1 < n) {
                        // S of the next block overwrites P after this PV has
                        // read it; its completion also covers this PV, so the
                        // softmax may then rescale O.
                        if (!(ok = mbar_wait_s(full_a + 8u * slot(idx), slot_par(idx), st))) break;
                        tc_fence_after();
                        mma_s(kdesc(idx));
                        umma_commit_s(sfull_a);
                        umma_commit_s(empty_a + 8u * slot(idx));
                        ++idx;
                        if (i + 2 == n) umma_commit_s(qempty_a);  // the tile's last S
                    }
                }
                if (!ok) break;
                umma_commit_s(ofinal_a);
                ++ni;
            }
            umma_commit(mma_done);
            mbar_wait_bounded(mma_done, 0);
        }
        __syncwarp();
      }
    } else {
        // ------------------------------------------------ softmax (warps 0-3)
        setmaxnreg_inc<T::REG_SOFTMAX>();
        const int r = warp * 32 + lane;  // row within the tile = TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
        const uint32_t s_tm = tmem + lane_off;
        const uint32_t o_tm = tmem + lane_off + T::O_COL;
        const float sl2 = p.scale_log2;
        // This warp's O staging box: bf16 [32 rows][64 columns], 128-byte
        // swizzle, TMA-stored one 64-column chunk at a time.
        uint8_t* stage = smem + T::OST_OFF + warp * T::OST_WARP;
        bool ok = true;
        int jb = 0, ni = 0;
        for (int it = blockIdx.x; it < items && ok; it += gridDim.x) {
            int qt, bh;
            decode(it, qt, bh);
            const int n = n_blocks(qt);
            const int row0 = qt * T::BM;
            const int row = row0 + r;
            float m = -INFINITY, l = 0.f, lr = 0.f;
            for (int j = 0; j < n; ++j, ++jb) {
                ok = __all_sync(0xffffffffu, mbar_wait(s_full, jb & 1, st));
                if (!ok) break;
                tc_fence_after();
                uint32_t sr[4][32];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(s_tm + 32u * c, sr[c]);
                tmem_ld_wait();
                const int kv0 = kv_block(n, j) * T::BN;
                const bool masked_block =
                    (kv0 + T::BN > N) || (CAUSAL && kv0 + T::BN - 1 > row0);
                if (masked_block) {
                    int lim = min(T::BN, N - kv0);
                    if (CAUSAL) lim = min(lim, row - kv0 + 1 - p.strict);
#pragma unroll
                    for (int c = 0; c < 128; ++c)
                        if (c >= lim) sr[c >> 5][c & 31] = __float_as_uint(-INFINITY);
                }
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
                const float m_blk = mx[0] * sl2;
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
                softmax_block_exp<T::PSPLIT>(sr, sl2, m == -INFINITY ? 0.f : m, s_tm, l, lr,
                                             p_half);
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(p_ready);
            }
            if (!ok) break;
            ok = __all_sync(0xffffffffu, mbar_wait(o_final, ni & 1, st));
            if (!ok) break;
            tc_fence_after();
            // A row with no visible key (strict causal row 0) keeps m = -inf:
            // O = 0, LSE = -inf.
            const float inv_l = m == -INFINITY ? 0.f : 1.0f / lr;
            const float lse_val = (m + log2f(l)) * 0.6931471805599453f;
            const int wrow0 = row0 + warp * 32;
#pragma unroll 1
            for (int c2 = 0; c2 < T::CHUNKS; ++c2) {
                uint32_t o[2][32];
                tmem_ld32(o_tm + 64u * c2, o[0]);
                tmem_ld32(o_tm + 64u * c2 + 32u, o[1]);
                tmem_ld_wait();
                if (c2 == T::CHUNKS - 1) {  // O is out of TMEM: the next tile's PV may start
                    tc_fence_before();
                    mbar_arrive(o_free);
                }
                if (lane == 0) bulk_wait_group_read0();  // the previous store has read the box
                __syncwarp();
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const uint32_t* a = o[u >> 2] + 8 * (u & 3);
                    uint4 v;
                    v.x = pack_bf16x2(__uint_as_float(a[0]) * inv_l, __uint_as_float(a[1]) * inv_l);
                    v.y = pack_bf16x2(__uint_as_float(a[2]) * inv_l, __uint_as_float(a[3]) * inv_l);
                    v.z = pack_bf16x2(__uint_as_float(a[4]) * inv_l, __uint_as_float(a[5]) * inv_l);
                    v.w = pack_bf16x2(__uint_as_float(a[6]) * inv_l, __uint_as_float(a[7]) * inv_l);
                    *reinterpret_cast<uint4*>(stage + sw128_offset(lane, u)) = v;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0 && wrow0 < N) {
                    tma_store_3d(&tmO, stage, c2 * 64, wrow0, bh);
                    bulk_commit_group();
                }
            }
            if (row < N) p.lse[static_cast<size_t>(bh) * N + row] = lse_val;
            ++ni;
        }
        if (lane == 0) bulk_wait_group0();  // every O store has completed
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
