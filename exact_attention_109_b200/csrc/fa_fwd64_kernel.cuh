// fa_fwd64_kernel.cuh -- the forward pass at d = 64 with two CTAs per SM.
//
// Same arithmetic as fa_fwd_kernel (FlashAttention-2 abstract; iplexlaw blog,
// "Tiling preserves the attention calculation": per query row an online
// softmax over key blocks, the partial output rescaled when the running
// maximum grows; exp2 with the scale folded in, deferred rescaling, every
// fourth pair of exponentials on the FMA pipe, O normalised by the sum of
// the bf16 weights the PV product used) and the same tile schedule: a CTA
// owns two 128-row query tiles of one head, and the tensor core alternates
// between them, computing one tile's PV and next scores while the softmax
// works on the other's.
//
// At d = 64 a key block costs half the MMA time of d = 128 but the same
// softmax work, and a CTA of fa_fwd_kernel spends ~1800 cycles per tile and
// 128-key block on ~770 cycles of exponentials and ~860 cycles of softmax
// instructions per SM sub-partition: it waits on latencies.  This kernel
// halves the key block to 64, so two tiles fit in 256 TMEM columns (S_t at
// [64t, 64t + 64) with P_t written back over its first 32 columns, O_t at
// [128 + 64t, 128 + 64t + 64)), and gives both tiles to one softmax
// warpgroup that alternates between them (thread r owns row r of both
// tiles).  A CTA then needs 256 threads and ~99 KB of shared memory, so two
// share an SM: four tiles in flight per SM instead of two.
//
// Roles: warps 0-3 the softmax (both tiles), warp 4 issues tcgen05.mma, warp
// 5 issues TMA, warps 6-7 idle.  K and V blocks ([64 keys][64 dims], 8 KB)
// alternate through a ring of slots under full/empty mbarriers; every wait is
// bounded.
#pragma once

#include "fa_fwd_kernel.cuh"

namespace fa {

struct Fwd64Traits {
    static constexpr int D = 64;
    static constexpr int BM = 128;                  // query rows per tile
    static constexpr int BN = 64;                   // key rows per block
    static constexpr int Q_TILE = BM * D * 2;       // 16 KB: [128 rows][128 B]
    static constexpr int KV_TILE = BN * D * 2;      // 8 KB: [64 rows][128 B]
    static constexpr int NSLOT = 8;
    static constexpr int Q_OFF = 0;
    static constexpr int KV_OFF = Q_OFF + 2 * Q_TILE;
    static constexpr int BAR_OFF = KV_OFF + NSLOT * KV_TILE;
    // q, full[NSLOT], empty[NSLOT], s_full[2], p_ready[2], o_final[2], mma_done
    static constexpr int NBAR = 1 + 2 * NSLOT + 2 + 2 + 2 + 1;
    static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
    static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;  // + alignment slack
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
    static constexpr float TAU = 8.0f;  // deferred-rescale threshold (log2 units)
    static_assert(2 * (SMEM_BYTES + 1024) <= 233472, "two CTAs per SM");
    static_assert(REG_BUDGET == NUM_THREADS * 128, "register split");
};

// One softmax row over a 64-key block (the 64-column counterpart of
// softmax_block_exp): p = exp2(s * scale*log2(e) - m) in f32x2 pairs, every
// fourth pair on the FMA pipe, packed to bf16 and written over the first 32
// TMEM columns of S; adds the fp32 sum of p to l and the sum of the
// bf16-rounded p to lr.
__device__ __forceinline__ void softmax_block64_exp(const uint32_t (&sr)[2][32], float sl2,
                                                    float m, uint32_t s_tm, float& l,
                                                    float& lr) {
    const uint64_t sl2x2 = f2_pack(sl2, sl2);
    const uint64_t negm2 = f2_pack(-m, -m);
    uint64_t sum2[2] = {0ull, 0ull};
    float rs[4] = {0.f, 0.f, 0.f, 0.f};
    uint32_t pk[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        const int c = 2 * e;
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
    tmem_st32(s_tm, pk);
    float a0, a1;
    f2_unpack(fadd2(sum2[0], sum2[1]), a0, a1);
    l += a0 + a1;
    lr += (rs[0] + rs[1]) + (rs[2] + rs[3]);
}

template <bool CAUSAL>
__global__ void __launch_bounds__(256, 2)
    fa_fwd64_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                    const FwdParams p) {
    using T = Fwd64Traits;
    constexpr int D = T::D;
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
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + T::MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + T::MISC_OFF + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // The tile pair schedule of fa_fwd_kernel: non-causal, a head's pairs
    // adjacent; causal, the heaviest pairs (the last of every head) first.
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
    // Key blocks (of 64) seen by each tile; causal tile t ends at key
    // q0 + 128t + 127, i.e. block 4qp + 2t + 1.
    const int n0 = CAUSAL ? min(n_kv, 4 * qp + 2) : n_kv;
    const int n1 = CAUSAL ? min(n_kv, 4 * qp + 4) : n_kv;
    // Causal: walked from the diagonal down, so tile 1's extra blocks come
    // first and both tiles end on block 0; tile 0 joins at iteration off0.
    const int off0 = n1 - n0;
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
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
        // Q and the first key/value block, requested before the TMEM
        // allocation and the block-wide sync so their latency overlaps both.
        mbar_arrive_expect_tx(bar_q, 2 * T::Q_TILE);
        for (int t = 0; t < 2; ++t)
            tma_load_3d(smem + T::Q_OFF + t * T::Q_TILE, &tmQ, bar_q, 0, q0 + 128 * t, bh);
        for (int h = 0; h < 2; ++h) {
            mbar_arrive_expect_tx(&full[h], T::KV_TILE);
            tma_load_3d(smem + T::KV_OFF + h * T::KV_TILE, h ? &tmV : &tmK, &full[h], 0,
                        kv_block(0) * T::BN, bh);
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
            int issued = 2;  // iteration 0's K and V were issued at set-up
            for (int j = 1; j < n1 && ok; ++j) {
                for (int h = 0; h < 2; ++h) {  // 0: K_j, 1: V_j
                    const int idx = 2 * j + h;
                    const int slot = idx % T::NSLOT;
                    if (!mbar_wait(&empty[slot], ((idx / T::NSLOT) & 1) ^ 1u, st)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[slot], T::KV_TILE);
                    tma_load_3d(smem + T::KV_OFF + slot * T::KV_TILE, h ? &tmV : &tmK,
                                &full[slot], 0, kv_block(j) * T::BN, bh);
                    ++issued;
                }
            }
            if (!ok) {  // let the copies already requested land before exiting
                for (int idx = max(0, issued - T::NSLOT); idx < issued; ++idx)
                    mbar_wait_bounded(&full[idx % T::NSLOT], (idx / T::NSLOT) & 1);
                mbar_wait_bounded(bar_q, 0);
            }
        }
        __syncwarp();
      } else if (warp == T::MMA_WARP) {
        // ------------------------------------------------ MMA issuer
        // This thread's instruction stream is on the kernel's critical path,
        // so descriptors and barrier addresses are built once and the ring
        // position advances by adds (as in fa_fwd_kernel).
        if (lane == 0) {
            const uint32_t q_base = smem_u32(smem + T::Q_OFF);
            const uint32_t kv_base = smem_u32(smem + T::KV_OFF);
            const uint64_t dq[2] = {sdesc_sw128(q_base, 16, 1024),
                                    sdesc_sw128(q_base + T::Q_TILE, 16, 1024)};
            const uint64_t dk_base = sdesc_sw128(kv_base, 16, 1024);        // K in slot 0
            const uint64_t dv_base = sdesc_sw128(kv_base, T::KV_TILE, 1024);  // V in slot 0
            const uint32_t full_a = smem_u32(full), empty_a = smem_u32(empty);
            const uint32_t sfull_a = smem_u32(s_full), pready_a = smem_u32(p_ready);
            const uint32_t ofinal_a = smem_u32(o_final);
            // S_t = Q_t K^T: M = 128, N = 64 keys, K = 64 dims, both K-major.
            auto mma_s = [&](int t, uint64_t dk0) {
                umma_ss_c<false>(tmem + 64u * t, dq[t], dk0, T::IDESC_S);
#pragma unroll
                for (int k = 1; k < D / 16; ++k)
                    umma_ss_c<true>(tmem + 64u * t, sdesc_add(dq[t], k * 32), sdesc_add(dk0, k * 32),
                                    T::IDESC_S);
            };
            // O_t += P_t V: M = 128, N = 64 dims, K = 64 keys; P from TMEM
            // (16 keys per 8 columns), V MN-major.
            auto mma_pv = [&](int t, uint64_t dv0, bool accumulate) {
                umma_ts(tmem + T::O_COL + 64u * t, tmem + 64u * t, dv0, T::IDESC_PV,
                        accumulate ? 1u : 0u);
#pragma unroll
                for (int k = 1; k < T::BN / 16; ++k)
                    umma_ts_c<true>(tmem + T::O_COL + 64u * t, tmem + 64u * t + 8u * k,
                                    sdesc_add(dv0, k * 2048), T::IDESC_PV);
            };
            auto pv_tile = [&](int t, uint64_t dv0, bool acc, uint32_t par) -> bool {
                if (!mbar_wait_s(pready_a + 8u * t, par, st)) return false;
                tc_fence_after();
                mma_pv(t, dv0, acc);
                return true;
            };
            // Tile 0 takes part in iterations [off0, n1) (off0 + n0 = n1).
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
            // Iteration j: PV_0(j-1), S_0(j), PV_1(j-1), S_1(j).  S of a tile
            // overwrites its P only after the PV that reads it (MMAs from
            // one thread run in order).  ks, kp: ring slot and phase parity
            // of K_j (position 2j); V_{j-1} sits one position before it.
            uint32_t ks = 2u % T::NSLOT, kp = (2u / T::NSLOT) & 1u;
            for (int j = 1; j < n1 && ok; ++j) {
                const uint32_t vs = ks ? ks - 1u : T::NSLOT - 1u;
                const uint32_t vp = ks ? kp : kp ^ 1u;
                ok = mbar_wait_s(full_a + 8u * ks, kp, st) && mbar_wait_s(full_a + 8u * vs, vp, st);
                if (!ok) break;
                tc_fence_after();
                const uint64_t dk = sdesc_add(dk_base, ks * T::KV_TILE);
                const uint64_t dv = sdesc_add(dv_base, vs * T::KV_TILE);
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
                const uint64_t dv = sdesc_add(dv_base, vs * T::KV_TILE);
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
        // ------------------------------------------------ softmax (both tiles)
        setmaxnreg_inc<T::REG_SOFTMAX>();
        const int r = warp * 32 + lane;  // row within each tile = TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
        const float sl2 = p.scale_log2;
        float m[2] = {-INFINITY, -INFINITY};  // reference maxima (log2 units)
        float l[2] = {0.f, 0.f};              // fp32 sums of the weights (LSE)
        float lr[2] = {0.f, 0.f};             // sums of the bf16 weights (O)
        int nb[2] = {0, 0};                   // blocks done per tile
        bool ok = true;
        // Block i of the walk: tile 0 (if it takes part) and then tile 1, in
        // the order the MMA warp produces their scores.
        for (int i = 0; i < n1 && ok; ++i) {
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                if (t == 0 && (i < off0 || i - off0 >= n0)) continue;
                const int j = nb[t];
                ok = __all_sync(0xffffffffu, mbar_wait(&s_full[t], j & 1, st));
                if (!ok) break;
                tc_fence_after();
                const uint32_t s_tm = tmem + lane_off + 64u * t;
                uint32_t sr[2][32];
                tmem_ld32(s_tm, sr[0]);
                tmem_ld32(s_tm + 32u, sr[1]);
                tmem_ld_wait();
                const int row0 = q0 + 128 * t;
                const int row = row0 + r;
                const int kv0 = kv_block(i) * T::BN;
                const bool masked_block =
                    (kv0 + T::BN > N) || (CAUSAL && kv0 + T::BN - 1 > row0);
                if (masked_block) {
                    int lim = min(T::BN, N - kv0);
                    if (CAUSAL) lim = min(lim, row - kv0 + 1 - p.strict);
#pragma unroll
                    for (int c = 0; c < 64; ++c)
                        if (c >= lim) sr[c >> 5][c & 31] = __float_as_uint(-INFINITY);
                }
                float mx[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) mx[q] = __uint_as_float(sr[0][q]);
#pragma unroll
                for (int c = 8; c < 64; c += 8)
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        mx[q] = fmaxf(mx[q], __uint_as_float(sr[(c + q) >> 5][(c + q) & 31]));
                mx[0] = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                              fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
                const float m_blk = mx[0] * sl2;
                const float m_new = (m_blk > m[t] + T::TAU) ? m_blk : m[t];
                if (j > 0) {
                    const bool grow = m_new != m[t];
                    if (__any_sync(0xffffffffu, grow)) {
                        const float alpha = grow ? ex2_approx(m[t] - m_new) : 1.0f;
                        l[t] *= alpha;
                        lr[t] *= alpha;
                        const uint32_t o_tm = tmem + lane_off + T::O_COL + 64u * t;
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
                m[t] = m_new;
                softmax_block64_exp(sr, sl2, m[t] == -INFINITY ? 0.f : m[t], s_tm, l[t], lr[t]);
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&p_ready[t]);
                ++nb[t];
            }
        }
        // Epilogue of each tile: O / lr as bf16, staged in the tile's Q
        // buffer (no MMA reads it any more), TMA-stored 32 rows per warp.
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            if (!ok) break;
            ok = __all_sync(0xffffffffu, mbar_wait(&o_final[t], 0, st));
            if (!ok) break;
            tc_fence_after();
            const int row0 = q0 + 128 * t;
            const int row = row0 + r;
            // A row with no visible key (strict causal row 0) keeps m = -inf:
            // O = 0, LSE = -inf.
            const float inv_l = m[t] == -INFINITY ? 0.f : 1.0f / lr[t];
            const float lse_val = (m[t] + log2f(l[t])) * 0.6931471805599453f;
            const uint32_t o_tm = tmem + lane_off + T::O_COL + 64u * t;
            uint32_t o[2][32];
            tmem_ld32(o_tm, o[0]);
            tmem_ld32(o_tm + 32u, o[1]);
            tmem_ld_wait();
            uint8_t* stage = smem + T::Q_OFF + t * T::Q_TILE + warp * 32 * 128;
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
            const int wrow0 = row0 + warp * 32;
            if (lane == 0 && wrow0 < N) {
                tma_store_3d(&tmO, stage, 0, wrow0, bh);
                bulk_commit_group();
            }
            if (row < N) p.lse[static_cast<size_t>(bh) * N + row] = lse_val;
        }
        if (lane == 0) bulk_wait_group_read0();
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
