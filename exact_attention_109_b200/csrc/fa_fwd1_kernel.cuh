// fa_fwd1_kernel.cuh -- the forward pass with one 128-row query tile per CTA,
// two CTAs per SM, for short sequences.
//
// Same arithmetic as fa_fwd_kernel (FlashAttention-2 abstract; iplexlaw blog,
// "Tiling preserves the attention calculation": per query row an online
// softmax over 128-key blocks, the partial output rescaled when the running
// maximum grows) and the same softmax code, but each CTA owns a single query
// tile and needs only 256 TMEM columns (S/P at [0, 128), O at [128, 128 + d))
// and about 100 KB of shared memory, so two CTAs share an SM.  When a
// sequence is short a CTA walks only a few key blocks, and the fixed cost
// of each CTA -- barrier and TMEM set-up, the first TMA round trip, the
// epilogue, the gap to the next CTA -- is as long as its work; with two CTAs
// per SM one CTA's fixed cost overlaps the other's MMAs and softmax (the
// blog's "Three changes improve GPU utilisation": keep the units busy at
// every sequence length).  The price is one S buffer per CTA: the score MMA
// of key block j+1 waits until the softmax of block j has written P, which
// the second CTA on the SM covers.
//
// Roles (256 threads = 2 warpgroups): warps 0-3 the softmax (one thread per
// query row = TMEM lane), warp 4 issues tcgen05.mma, warp 5 issues TMA, warps
// 6-7 idle.  K and V alternate through a ring of slots (K_j in slot 2j, V_j in
// 2j+1, modulo the ring) under full/empty mbarriers; every wait is bounded.
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
    static constexpr int BAR_OFF = KV_OFF + NSLOT * TILE_BYTES;
    // q, full[NSLOT], empty[NSLOT], s_full, p_ready, p_half, o_final, mma_done
    static constexpr int NBAR = 1 + 2 * NSLOT + 5;
    static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
    static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;
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
    static_assert(2 * (SMEM_BYTES + 1024) <= 233472, "two CTAs per SM");
};

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(256, 2)
    fa_fwd1_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                   const FwdParams p) {
    using T = Fwd1Traits<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::BAR_OFF);
    uint64_t* bar_q = bars;
    uint64_t* full = bars + 1;
    uint64_t* empty = full + T::NSLOT;
    uint64_t* s_full = empty + T::NSLOT;
    uint64_t* p_ready = s_full + 1;
    uint64_t* p_half = p_ready + 1;
    uint64_t* o_final = p_half + 1;
    uint64_t* mma_done = o_final + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + T::MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + T::MISC_OFF + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // Query tile qt of head bh.  Causal: the last tiles of every head (most
    // key blocks) first; non-causal: a head's tiles adjacent (K/V reuse in L2).
    const int N = p.N;
    const int n_qt = (N + T::BM - 1) / T::BM;
    int qt, bh;
    if (CAUSAL) {
        bh = static_cast<int>(blockIdx.x % p.bh_count);
        qt = n_qt - 1 - static_cast<int>(blockIdx.x / p.bh_count);
    } else {
        qt = static_cast<int>(blockIdx.x % n_qt);
        bh = static_cast<int>(blockIdx.x / n_qt);
    }
    const int row0 = qt * T::BM;
    const int n_kv = (N + T::BN - 1) / T::BN;
    const int n = CAUSAL ? min(n_kv, qt + 1) : n_kv;   // key blocks of this tile
    // causal: from the diagonal down, so the masked block comes first
    auto kv_block = [&](int i) { return CAUSAL ? n - 1 - i : i; };

    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        for (int s = 0; s < T::NSLOT; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(s_full, 1);
        mbar_init(p_ready, 128);
        mbar_init(p_half, 128);
        mbar_init(o_final, 1);
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
        // Q and the first key/value block, requested before the TMEM
        // allocation and the block-wide sync so their latency overlaps both.
        mbar_arrive_expect_tx(bar_q, T::TILE_BYTES);
        for (int c = 0; c < T::CHUNKS; ++c)
            tma_load_3d(smem + T::Q_OFF + c * T::CHUNK_BYTES, &tmQ, bar_q, c * 64, row0, bh);
        for (int h = 0; h < 2; ++h) {
            mbar_arrive_expect_tx(&full[h], T::TILE_BYTES);
            for (int c = 0; c < T::CHUNKS; ++c)
                tma_load_3d(smem + T::KV_OFF + h * T::TILE_BYTES + c * T::CHUNK_BYTES,
                            h ? &tmV : &tmK, &full[h], c * 64, kv_block(0) * T::BN, bh);
        }
    }
    if (warp == T::MMA_WARP) {
        tmem_alloc(tmem_slot, T::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == T::LOAD_WARP && lane == 0) {
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
            int issued = 2;
            for (int j = 1; j < n && ok; ++j) {
                for (int h = 0; h < 2; ++h) {  // 0: K_j, 1: V_j
                    const int idx = 2 * j + h;
                    const int slot = idx % T::NSLOT;
                    if (!mbar_wait(&empty[slot], ((idx / T::NSLOT) & 1) ^ 1u, st)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[slot], T::TILE_BYTES);
                    for (int c = 0; c < T::CHUNKS; ++c)
                        tma_load_3d(smem + T::KV_OFF + slot * T::TILE_BYTES + c * T::CHUNK_BYTES,
                                    h ? &tmV : &tmK, &full[slot], c * 64, kv_block(j) * T::BN,
                                    bh);
                    ++issued;
                }
            }
            if (!ok) {
                for (int idx = max(0, issued - T::NSLOT); idx < issued; ++idx)
                    mbar_wait_bounded(&full[idx % T::NSLOT], (idx / T::NSLOT) & 1);
                mbar_wait_bounded(bar_q, 0);
            }
        }
        __syncwarp();
      } else if (warp == T::MMA_WARP) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t q_base = smem_u32(smem + T::Q_OFF);
            const uint32_t kv_base = smem_u32(smem + T::KV_OFF);
            auto slot_addr = [&](int idx) {
                return kv_base + static_cast<uint32_t>((idx % T::NSLOT) * T::TILE_BYTES);
            };
            auto slot_par = [&](int idx) { return static_cast<uint32_t>((idx / T::NSLOT) & 1); };
            const uint64_t dq0 = sdesc_sw128(q_base, 16, 1024);
            // S = Q K^T: M=128, N=128, K=D, both K-major.
            auto mma_s = [&](uint32_t k_addr) {
                const uint64_t dk0 = sdesc_sw128(k_addr, 16, 1024);
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
            auto mma_pv = [&](uint32_t v_addr, bool accumulate, int k0, int k1) {
                const uint64_t dv0 = sdesc_sw128(v_addr, T::CHUNK_BYTES, 1024);
#pragma unroll
                for (int k = k0; k < k1; ++k) {
                    if (k == 0)
                        umma_ts(tmem + T::O_COL, tmem, dv0, T::IDESC_PV, accumulate ? 1u : 0u);
                    else
                        umma_ts_c<true>(tmem + T::O_COL, tmem + 8u * k, sdesc_add(dv0, k * 2048),
                                        T::IDESC_PV);
                }
            };
            bool ok = mbar_wait(bar_q, 0, st) && mbar_wait(&full[0], 0, st);
            if (ok) {
                tc_fence_after();
                mma_s(slot_addr(0));
                umma_commit(s_full);
                umma_commit(&empty[0]);
            }
            for (int i = 0; i < n && ok; ++i) {
                const int iv = 2 * i + 1, ik = 2 * i + 2;  // V of block i, K of block i + 1
                const uint32_t par = i & 1;
                ok = mbar_wait(&full[iv % T::NSLOT], slot_par(iv), st);
                if (!ok) break;
                if constexpr (T::PSPLIT) {
                    if (!(ok = mbar_wait(p_half, par, st))) break;
                    tc_fence_after();
                    mma_pv(slot_addr(iv), i > 0, 0, T::BN / 32);
                    if (!(ok = mbar_wait(p_ready, par, st))) break;
                    tc_fence_after();
                    mma_pv(slot_addr(iv), true, T::BN / 32, T::BN / 16);
                } else {
                    if (!(ok = mbar_wait(p_ready, par, st))) break;
                    tc_fence_after();
                    mma_pv(slot_addr(iv), i > 0, 0, T::BN / 16);
                }
                umma_commit(&empty[iv % T::NSLOT]);
                if (i + 1 < n) {
                    // S of the next block overwrites P in TMEM after this PV
                    // has read it (MMAs from one thread run in order); its
                    // completion also covers this PV, so the softmax may
                    // then rescale O.
                    if (!(ok = mbar_wait(&full[ik % T::NSLOT], slot_par(ik), st))) break;
                    tc_fence_after();
                    mma_s(slot_addr(ik));
                    umma_commit(s_full);
                    umma_commit(&empty[ik % T::NSLOT]);
                }
            }
            if (ok) umma_commit(o_final);
            umma_commit(mma_done);
            mbar_wait_bounded(mma_done, 0);
        }
        __syncwarp();
      }
    } else {
        // ------------------------------------------------ softmax (warps 0-3)
        setmaxnreg_inc<T::REG_SOFTMAX>();
        const int r = warp * 32 + lane;  // row within the tile = TMEM lane
        const int row = row0 + r;
        const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
        const uint32_t s_tm = tmem + lane_off;
        const uint32_t o_tm = tmem + lane_off + T::O_COL;
        const float sl2 = p.scale_log2;
        float m = -INFINITY, l = 0.f, lr = 0.f;
        bool ok = true;
        for (int j = 0; j < n; ++j) {
            ok = __all_sync(0xffffffffu, mbar_wait(s_full, j & 1, st));
            if (!ok) break;
            tc_fence_after();
            uint32_t sr[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(s_tm + 32u * c, sr[c]);
            tmem_ld_wait();
            const int kv0 = kv_block(j) * T::BN;
            const bool masked_block = (kv0 + T::BN > N) || (CAUSAL && kv0 + T::BN - 1 > row0);
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
            softmax_block_exp<T::PSPLIT>(sr, sl2, m == -INFINITY ? 0.f : m, s_tm, l, lr, p_half);
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(p_ready);
        }
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(o_final, 0, st));
        if (ok) {
            tc_fence_after();
            const float inv_l = m == -INFINITY ? 0.f : 1.0f / lr;
            const float lse_val = (m + log2f(l)) * 0.6931471805599453f;
            // O (bf16, 128-byte swizzle) staged in the Q buffer, which no MMA
            // reads any more; TMA-stored 32 rows per warp.
            uint8_t* stage = smem + T::Q_OFF + warp * 32 * 128;
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
            const int wrow0 = row0 + warp * 32;
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
