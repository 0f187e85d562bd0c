// fa_bwd64_kernel.cuh -- the backward main stage at d = 64 with two CTAs
// per SM.
//
// Same arithmetic and workspace as fa_bwd_main_kernel (the textbook gradient
// of softmax attention, recomputed tile by tile as the FlashAttention-2
// abstract and the iplexlaw blog, "Tiling preserves the attention
// calculation", describe): one CTA per (batch*head, 128-row key block j)
// with K_j and V_j resident, walking the 64-row query blocks (causal: from
// the diagonal), recomputing S^T = K Q^T and dP^T = V dO^T, forming P and dS,
// and accumulating dV += P^T dO, dK += dS^T Q, dQ += dS K.
//
// What differs is the footprint.  At d = 64 one block's work is a chain of
// small steps -- 8 score MMAs, the P/dS math, 16 gradient MMAs, the dQ
// drain -- whose latencies the tensor core cannot hide within one CTA: the
// 64-row kernel spends ~2900 cycles per block on ~1150 cycles of MMAs.  This
// kernel keeps one block in flight per CTA and makes the CTA small enough
// that two share an SM, so one CTA's MMAs fill the other's gaps:
//   * TMEM, 256 columns: S^T at [0, 64) (P^T written back over its first 32
//     columns as bf16), dP^T at [64, 128) (dS^T over its first 32 columns,
//     then dQ^T), dV at [128, 192), dK at [192, 256);
//   * shared memory, ~99 KB: K, V, two Q/dO stages, one dS^T tile, the dQ
//     staging boxes;
//   * 256 threads: warps 0-3 the P/dS warpgroup (one thread per key row, all
//     64 query columns in two halves), warps 4-5 the dQ drain (TMEM lanes
//     0-63 = head dims), warp 6 the MMA issuer, warp 7 the TMA producer.
// Every wait is bounded.
#pragma once

#include "fa_bwd_kernels.cuh"

namespace fa {

struct Bwd64Traits {
    static constexpr int D = 64;
    static constexpr int BN = 128;                // key rows per CTA
    static constexpr int BM = 64;                 // query rows per block
    static constexpr int KV_TILE = BN * D * 2;    // 16 KB: [128 rows][128 B]
    static constexpr int Q_TILE = BM * D * 2;     // 8 KB: [64 rows][128 B]
    static constexpr int NSTAGE = 2;
    static constexpr int STAGE_BYTES = 2 * Q_TILE;  // Q_i then dO_i
    static constexpr int DS_TILE = BN * BM * 2;     // dS^T [128 keys][64 queries] bf16
    static constexpr int DQ_WARP_BYTES = BM * 128;  // fp32 [64 q][32 d] per drain warp
    static constexpr int K_OFF = 0;
    static constexpr int V_OFF = K_OFF + KV_TILE;   // V follows K directly
    static constexpr int ST_OFF = V_OFF + KV_TILE;
    static constexpr int DS_OFF = ST_OFF + NSTAGE * STAGE_BYTES;
    static constexpr int DQ_OFF = DS_OFF + DS_TILE;
    static constexpr int VEC_OFF = DQ_OFF + 2 * DQ_WARP_BYTES;  // lse2, dvec per stage
    static constexpr int BAR_OFF = VEC_OFF + NSTAGE * 2 * BM * 4;
    // kv, stage_full[NS], stage_empty[NS], sdp_full, pds_ready, dq_full,
    // dq_drained, kv_done, mma_done
    static constexpr int NBAR = 1 + 2 * NSTAGE + 6;
    static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
    // No alignment slack: the kernel checks that the dynamic shared memory
    // starts on a 1024-byte boundary and reports kErrLayout if not.
    static constexpr int SMEM_BYTES = MISC_OFF + 16;
    static constexpr int NUM_THREADS = 256;
    static constexpr int DRAIN_WARP0 = 4;
    static constexpr int MMA_WARP = 6;
    static constexpr int LOAD_WARP = 7;
    static constexpr uint32_t REG_COMPUTE = 168;
    static constexpr uint32_t REG_OTHER = 88;
    static constexpr int REG_BUDGET = 128 * (REG_COMPUTE + REG_OTHER);
    static constexpr uint32_t TMEM_COLS = 256;
    static constexpr uint32_t S_COL = 0;
    static constexpr uint32_t DP_COL = 64;
    static constexpr uint32_t DV_COL = 128;
    static constexpr uint32_t DK_COL = 192;
    static constexpr uint32_t IDESC_SDP = idesc_bf16_f32(128, BM, 0, 0);
    static constexpr uint32_t IDESC_ACC = idesc_bf16_f32(128, D, 0, 1);
    static constexpr uint32_t IDESC_DQ = idesc_bf16_f32(128, BM, 1, 1);
    static_assert(2 * (SMEM_BYTES + 1024) <= 233472, "two CTAs per SM");
    static_assert(REG_BUDGET == NUM_THREADS * 128, "register split");
    // The epilogue stages dV / dK in the stage ring, which no MMA reads then:
    // bf16 [32 rows][64 columns] or two fp32 [32][32] boxes per warp.
    static_assert(4 * 2 * 4096 <= NSTAGE * STAGE_BYTES, "epilogue staging");
};

template <bool CAUSAL>
__global__ void __launch_bounds__(256, 2) fa_bwd_main64_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
    const __grid_constant__ CUtensorMap tmdK, const __grid_constant__ CUtensorMap tmdV,
    const __grid_constant__ CUtensorMap tmAcc, const BwdParams p) {
    using T = Bwd64Traits;
    constexpr int D = T::D;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw;
    if (smem_u32(smem) & 1023u) {  // the same for every thread of the block
        if (threadIdx.x == 0) atomicOr(p.err, kErrLayout);
        return;
    }

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::BAR_OFF);
    uint64_t* bar_kv = bars;
    uint64_t* stage_full = bars + 1;
    uint64_t* stage_empty = stage_full + T::NSTAGE;
    uint64_t* sdp_full = stage_empty + T::NSTAGE;
    uint64_t* pds_ready = sdp_full + 1;
    uint64_t* dq_full = pds_ready + 1;
    uint64_t* dq_drained = dq_full + 1;
    uint64_t* kv_done = dq_drained + 1;
    uint64_t* mma_done = kv_done + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + T::MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + T::MISC_OFF + 4);
    float* vec = reinterpret_cast<float*>(smem + T::VEC_OFF);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // Key block j of head bh, in the order of fa_bwd_main_kernel.
    int j, bh;
    if (CAUSAL) {
        j = static_cast<int>(blockIdx.x / p.bh_count);
        bh = static_cast<int>(blockIdx.x % p.bh_count);
    } else {
        j = static_cast<int>(blockIdx.x % p.n_kv);
        bh = static_cast<int>(blockIdx.x / p.n_kv);
    }
    const int N = p.N;
    const int qb0 = CAUSAL ? 2 * j : 0;   // first query block at/below the diagonal
    const int n = p.n_q - qb0;            // query blocks this CTA walks (>= 1)

    if (threadIdx.x == 0) {
        mbar_init(bar_kv, 1);
        for (int s = 0; s < T::NSTAGE; ++s) {
            mbar_init(&stage_full[s], 1);
            mbar_init(&stage_empty[s], 1);
        }
        mbar_init(sdp_full, 1);
        mbar_init(pds_ready, 128);
        mbar_init(dq_full, 1);
        mbar_init(dq_drained, 64);
        mbar_init(kv_done, 1);
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
        tma_prefetch_desc(&tmdO);
        tma_prefetch_desc(&tmAcc);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const AbortState st{abort_flag, p.err};
    if (warp >= T::DRAIN_WARP0) {
      setmaxnreg_dec<T::REG_OTHER>();
      if (warp == T::LOAD_WARP) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            bool ok = true;
            mbar_arrive_expect_tx(bar_kv, 2 * T::KV_TILE);
            tma_load_3d(smem + T::K_OFF, &tmK, bar_kv, 0, j * T::BN, bh);
            tma_load_3d(smem + T::V_OFF, &tmV, bar_kv, 0, j * T::BN, bh);
            int issued = 0;
            for (int k = 0; k < n; ++k) {
                const int s = k % T::NSTAGE;
                if (!mbar_wait(&stage_empty[s], ((k / T::NSTAGE) & 1) ^ 1u, st)) {
                    ok = false;
                    break;
                }
                const int qrow = (qb0 + k) * T::BM;
                uint8_t* sq = smem + T::ST_OFF + s * T::STAGE_BYTES;
                mbar_arrive_expect_tx(&stage_full[s], T::STAGE_BYTES + 2 * T::BM * 4);
                tma_load_3d(sq, &tmQ, &stage_full[s], 0, qrow, bh);
                tma_load_3d(sq + T::Q_TILE, &tmdO, &stage_full[s], 0, qrow, bh);
                const size_t voff = static_cast<size_t>(bh) * p.n_pad + qrow;
                bulk_load(vec + s * 2 * T::BM, p.lse2 + voff, T::BM * 4, &stage_full[s]);
                bulk_load(vec + s * 2 * T::BM + T::BM, p.dvec + voff, T::BM * 4, &stage_full[s]);
                ++issued;
            }
            if (!ok) {  // let the copies already requested land before exiting
                for (int k = max(0, issued - T::NSTAGE); k < issued; ++k)
                    mbar_wait_bounded(&stage_full[k % T::NSTAGE], (k / T::NSTAGE) & 1);
                mbar_wait_bounded(bar_kv, 0);
            }
        }
        __syncwarp();
      } else if (warp == T::MMA_WARP) {
        // ------------------------------------------------ MMA issuer
        // This thread paces the kernel, so the stage descriptors and barrier
        // addresses are built once and the stage ring advances by adds.
        if (lane == 0) {
            const uint32_t k_base = smem_u32(smem + T::K_OFF);
            const uint32_t st_base = smem_u32(smem + T::ST_OFF);
            // Stage 0's Q and dO, K-major (S^T, dP^T) and MN-major (dV, dK);
            // stage s adds s * STAGE_BYTES.
            const uint64_t sq_k = sdesc_sw128(st_base, 16, 1024);
            const uint64_t sdo_k = sdesc_sw128(st_base + T::Q_TILE, 16, 1024);
            const uint64_t sq_mn = sdesc_sw128(st_base, T::Q_TILE, 1024);
            const uint64_t sdo_mn = sdesc_sw128(st_base + T::Q_TILE, T::Q_TILE, 1024);
            const uint32_t sfull_a = smem_u32(stage_full), sempty_a = smem_u32(stage_empty);
            const uint32_t sdpf_a = smem_u32(sdp_full), pds_a = smem_u32(pds_ready);
            const uint32_t dqf_a = smem_u32(dq_full), dqd_a = smem_u32(dq_drained);
            const uint64_t dk0 = sdesc_sw128(k_base, 16, 1024);
            const uint64_t dv0 = sdesc_sw128(smem_u32(smem + T::V_OFF), 16, 1024);
            // K^T as the A operand of dQ^T, MN-major: M = 128 rows of which
            // the first 64 are the head dims (the other 64 lanes read the V
            // tile behind K and are never drained).
            const uint64_t dkt0 = sdesc_sw128(k_base, T::KV_TILE, 1024);
            const uint64_t dds0 = sdesc_sw128(smem_u32(smem + T::DS_OFF), T::DS_TILE, 1024);
            // S^T = K Q^T into [0, 64) and dP^T = V dO^T into [64, 128):
            // M = 128 keys, N = 64 queries, K = 64 head dims.
            auto mma_sdp = [&](uint32_t soff) {  // soff: the stage's byte offset
                const uint64_t dq0 = sdesc_add(sq_k, soff);
                const uint64_t ddo0 = sdesc_add(sdo_k, soff);
                umma_ss_c<false>(tmem + T::S_COL, dk0, dq0, T::IDESC_SDP);
#pragma unroll
                for (int kk = 1; kk < D / 16; ++kk)
                    umma_ss_c<true>(tmem + T::S_COL, sdesc_add(dk0, kk * 32), sdesc_add(dq0, kk * 32),
                                    T::IDESC_SDP);
                umma_ss_c<false>(tmem + T::DP_COL, dv0, ddo0, T::IDESC_SDP);
#pragma unroll
                for (int kk = 1; kk < D / 16; ++kk)
                    umma_ss_c<true>(tmem + T::DP_COL, sdesc_add(dv0, kk * 32),
                                    sdesc_add(ddo0, kk * 32), T::IDESC_SDP);
            };
            // dV += P^T dO and dK += dS^T Q: M = 128 keys, N = 64 head dims,
            // K = 64 queries; A (P^T at [0, 32), dS^T at [64, 96)) from TMEM,
            // B (dO or Q) MN-major from the stage.
            auto mma_dkdv = [&](uint32_t soff, bool first) {
                const uint64_t bq0 = sdesc_add(sq_mn, soff);
                const uint64_t bdo0 = sdesc_add(sdo_mn, soff);
                const uint32_t acc = first ? 0u : 1u;  // the first block overwrites
                umma_ts(tmem + T::DV_COL, tmem + T::S_COL, bdo0, T::IDESC_ACC, acc);
                umma_ts(tmem + T::DK_COL, tmem + T::DP_COL, bq0, T::IDESC_ACC, acc);
#pragma unroll
                for (int kk = 1; kk < T::BM / 16; ++kk) {
                    umma_ts_c<true>(tmem + T::DV_COL, tmem + T::S_COL + 8u * kk,
                                    sdesc_add(bdo0, kk * 2048), T::IDESC_ACC);
                    umma_ts_c<true>(tmem + T::DK_COL, tmem + T::DP_COL + 8u * kk,
                                    sdesc_add(bq0, kk * 2048), T::IDESC_ACC);
                }
            };
            // dQ^T = K^T dS^T into [64, 128): M = 128 (head dims; rows >= 64
            // unused), N = 64 queries, K = 128 keys; both MN-major.
            auto mma_dq = [&]() {
                umma_ss_c<false>(tmem + T::DP_COL, dkt0, dds0, T::IDESC_DQ);
#pragma unroll
                for (int kk = 1; kk < T::BN / 16; ++kk)
                    umma_ss_c<true>(tmem + T::DP_COL, sdesc_add(dkt0, kk * 2048),
                                    sdesc_add(dds0, kk * 2048), T::IDESC_DQ);
            };
            bool ok = mbar_wait(bar_kv, 0, st) && mbar_wait_s(sfull_a, 0, st);
            if (ok) {
                tc_fence_after();
                mma_sdp(0);
                umma_commit_s(sdpf_a);
            }
            // Stage slot of block k (s0) and of block k+1 (s1, with its
            // phase parity p1), advanced by one slot per block.
            uint32_t s0 = 0, s1 = 1u % T::NSTAGE, p1 = (1u / T::NSTAGE) & 1u;
            for (int k = 0; k < n && ok; ++k) {
                if (!(ok = mbar_wait_s(pds_a, k & 1, st))) break;
                tc_fence_after();
                mma_dkdv(s0 * T::STAGE_BYTES, k == 0);
                // dQ^T takes the dP^T columns after dK above has read dS^T
                // from them (MMAs from one thread run in order).
                mma_dq();
                umma_commit_s(dqf_a);
                umma_commit_s(sempty_a + 8u * s0);
                if (k + 1 < n) {
                    // S^T(k+1) overwrites P^T(k) after dV(k) has read it (in
                    // order); dP^T(k+1) waits for the drain to have read
                    // dQ^T(k).  Their commit also covers dQ^T(k), the last
                    // reader of the dS^T tile that block k+1 rewrites.
                    if (!(ok = mbar_wait_s(sfull_a + 8u * s1, p1, st))) break;
                    if (!(ok = mbar_wait_s(dqd_a, k & 1, st))) break;
                    tc_fence_after();
                    mma_sdp(s1 * T::STAGE_BYTES);
                    umma_commit_s(sdpf_a);
                }
                if (++s0 == T::NSTAGE) s0 = 0;
                if (++s1 == T::NSTAGE) {
                    s1 = 0;
                    p1 ^= 1u;
                }
            }
            if (ok) umma_commit(kv_done);
            umma_commit(mma_done);
            mbar_wait_bounded(mma_done, 0);
        }
        __syncwarp();
      } else {
        // ------------------------------------------------ dQ drain (warps 4-5)
        const int lg = warp - T::DRAIN_WARP0;  // TMEM lanes [32 lg, 32 lg + 32) = head dims
        const uint32_t dq_tm = tmem + (static_cast<uint32_t>(lg * 32) << 16) + T::DP_COL;
        uint8_t* buf = smem + T::DQ_OFF + lg * T::DQ_WARP_BYTES;
        for (int k = 0; k < n; ++k) {
            if (!__all_sync(0xffffffffu, mbar_wait(dq_full, k & 1, st))) break;
            tc_fence_after();
            uint32_t a[2][32];
            tmem_ld32(dq_tm, a[0]);
            tmem_ld32(dq_tm + 32u, a[1]);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(dq_drained);
            if (lane == 0) bulk_wait_group_read0();  // the previous reduce has read buf
            __syncwarp();
            // fp32 box [64 queries][32 head dims], 128-byte swizzle.
#pragma unroll
            for (int q = 0; q < T::BM; ++q)
                *reinterpret_cast<float*>(buf + q * 128 + ((((lane >> 2) ^ (q & 7))) << 4) +
                                          (lane & 3) * 4) = __uint_as_float(a[q >> 5][q & 31]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                tma_reduce_add_3d(&tmAcc, buf, lg * 32, (qb0 + k) * T::BM, bh);
                bulk_commit_group();
            }
        }
        if (lane == 0) bulk_wait_group0();
        __syncwarp();
      }
    } else {
        // ------------------------------------------------ P / dS (one thread per key row)
        setmaxnreg_inc<T::REG_COMPUTE>();
        const int r = warp * 32 + lane;
        const int kv_row = j * T::BN + r;
        const bool row_live = kv_row < N;  // rows past N: P = 0 (their K, V are zero-filled)
        const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
        const uint32_t s_tm = tmem + lane_off + T::S_COL;
        const uint32_t dp_tm = tmem + lane_off + T::DP_COL;
        const float sl2 = p.scale_log2;
        uint8_t* dsrow = smem + T::DS_OFF;
        bool ok = true;
        for (int k = 0; k < n; ++k) {
            ok = __all_sync(0xffffffffu, mbar_wait(sdp_full, k & 1, st));
            if (!ok) break;
            tc_fence_after();
            const float* vk = vec + (k % T::NSTAGE) * 2 * T::BM;
            // Two halves of 32 query columns.  Half h writes P^T over S
            // columns [16h, 16h + 16) and dS^T over dP columns [16h, 16h + 16),
            // both among the columns half 0 has already read.
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t sv[32], dp[32];
                tmem_ld32(s_tm + 32u * h, sv);
                tmem_ld32(dp_tm + 32u * h, dp);
                tmem_ld_wait();
                const float4* l4 = reinterpret_cast<const float4*>(vk + 32 * h);
                const float4* d4 = reinterpret_cast<const float4*>(vk + T::BM + 32 * h);
                const int qrow0 = (qb0 + k) * T::BM + 32 * h;
                // columns e < masked are hidden (strict: the diagonal too)
                const int masked = CAUSAL ? kv_row - qrow0 + p.strict : 0;
                uint32_t pk[16], dk[16];
#pragma unroll
                for (int e4 = 0; e4 < 8; ++e4) {
                    const float4 lv = l4[e4];
                    const float4 dvv = d4[e4];
                    const float lsv[4] = {lv.x, lv.y, lv.z, lv.w};
                    const float dsv_[4] = {dvv.x, dvv.y, dvv.z, dvv.w};
                    float pr[4], ds[4];
#pragma unroll
                    for (int hh = 0; hh < 4; ++hh) {
                        const int e = 4 * e4 + hh;
                        float x = ex2_approx(fmaf(__uint_as_float(sv[e]), sl2, -lsv[hh]));
                        if (!row_live || (CAUSAL && e < masked)) x = 0.f;
                        pr[hh] = x;
                        ds[hh] = x * (__uint_as_float(dp[e]) - dsv_[hh]);
                    }
                    pk[2 * e4] = pack_bf16x2(pr[0], pr[1]);
                    pk[2 * e4 + 1] = pack_bf16x2(pr[2], pr[3]);
                    dk[2 * e4] = pack_bf16x2(ds[0], ds[1]);
                    dk[2 * e4 + 1] = pack_bf16x2(ds[2], ds[3]);
                }
                tmem_st16(s_tm + 16u * h, pk);
                tmem_st16(dp_tm + 16u * h, dk);
                // dS^T row r, queries [32h, 32h + 32): four 16-byte units of
                // the 128-byte-swizzled tile (B operand of dQ^T).
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    *reinterpret_cast<uint4*>(dsrow + sw128_offset(r, 4 * h + u)) =
                        make_uint4(dk[4 * u], dk[4 * u + 1], dk[4 * u + 2], dk[4 * u + 3]);
            }
            fence_proxy_async_smem();
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(pds_ready);
        }
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(kv_done, 0, st));
        const int wrow0 = j * T::BN + warp * 32;
        if (ok && p.accum) {
            // Accumulating: dV, then scale*dK, added to fp32 [B*H][N][D]
            // buffers with TMA bulk reduce-adds of [32 rows][32 head dims]
            // boxes, staged two per warp in the stage ring.
            tc_fence_after();
            uint8_t* stage = smem + T::ST_OFF + warp * 2 * 4096;
#pragma unroll 1
            for (int c = 0; c < 2 * D / 32; ++c) {
                const bool is_dk = c >= D / 32;
                const uint32_t col = (is_dk ? T::DK_COL : T::DV_COL) + 32u * (c % (D / 32));
                const float mul = is_dk ? p.scale : 1.0f;
                uint32_t a[32];
                tmem_ld32(tmem + lane_off + col, a);
                tmem_ld_wait();
                uint8_t* box = stage + (c & 1) * 4096;
                if (c >= 2) {
                    if (lane == 0) bulk_wait_group_read<1>();  // box c-2 was read
                    __syncwarp();
                }
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    *reinterpret_cast<float4*>(box + sw128_offset(lane, u)) =
                        make_float4(__uint_as_float(a[4 * u + 0]) * mul,
                                    __uint_as_float(a[4 * u + 1]) * mul,
                                    __uint_as_float(a[4 * u + 2]) * mul,
                                    __uint_as_float(a[4 * u + 3]) * mul);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0 && wrow0 < N) {
                    tma_reduce_add_3d(is_dk ? &tmdK : &tmdV, box, 32 * (c % (D / 32)), wrow0, bh);
                    bulk_commit_group();
                }
            }
            if (lane == 0 && wrow0 < N) bulk_wait_group0();
        } else if (ok) {
            // dV, then scale*dK: bf16 [32 rows][64 head dims] per warp,
            // 128-byte swizzle, staged in the stage ring and TMA-stored.
            tc_fence_after();
#pragma unroll 1
            for (int g = 0; g < 2; ++g) {
                const uint32_t col0 = g ? T::DK_COL : T::DV_COL;
                const float mul = g ? p.scale : 1.0f;
                uint8_t* stage = smem + T::ST_OFF + (g * 4 + warp) * 4096;
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t a[32];
                    tmem_ld32(tmem + lane_off + col0 + 32u * c, a);
                    tmem_ld_wait();
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        uint4 v;
                        v.x = pack_bf16x2(__uint_as_float(a[8 * u + 0]) * mul,
                                          __uint_as_float(a[8 * u + 1]) * mul);
                        v.y = pack_bf16x2(__uint_as_float(a[8 * u + 2]) * mul,
                                          __uint_as_float(a[8 * u + 3]) * mul);
                        v.z = pack_bf16x2(__uint_as_float(a[8 * u + 4]) * mul,
                                          __uint_as_float(a[8 * u + 5]) * mul);
                        v.w = pack_bf16x2(__uint_as_float(a[8 * u + 6]) * mul,
                                          __uint_as_float(a[8 * u + 7]) * mul);
                        *reinterpret_cast<uint4*>(stage + sw128_offset(lane, 4 * c + u)) = v;
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0 && wrow0 < N) {
                    tma_store_3d(g ? &tmdK : &tmdV, stage, 0, wrow0, bh);
                    bulk_commit_group();
                }
            }
            if (lane == 0 && wrow0 < N) bulk_wait_group_read0();
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

// Stage 2 at d = 64 with two CTAs per SM (needs stage 1's workspace).  The
// maps are those of launch_bwd_main at d = 64.
template <bool CAUSAL>
cudaError_t launch_bwd_main64(int bh, int N, float scale, const BwdWorkspace& ws,
                              const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                              const CUtensorMap& mdo, const CUtensorMap& mdk,
                              const CUtensorMap& mdv, const CUtensorMap& macc, unsigned int* err,
                              cudaStream_t s, int accum, int strict) {
    using T = Bwd64Traits;
    BwdParams prm{};
    prm.lse2 = ws.lse2;
    prm.dvec = ws.dvec;
    prm.err = err;
    prm.N = N;
    prm.n_pad = ws.n_pad;
    prm.bh_count = bh;
    prm.n_kv = (N + T::BN - 1) / T::BN;
    prm.n_q = (N + T::BM - 1) / T::BM;
    prm.accum = accum;
    prm.H = 1;
    prm.scale = scale;
    prm.scale_log2 = scale * 1.4426950408889634f;
    prm.strict = strict;
    const long long grid = static_cast<long long>(bh) * prm.n_kv;
    fa_bwd_main64_kernel<CAUSAL><<<static_cast<unsigned>(grid), T::NUM_THREADS, T::SMEM_BYTES,
                                   s>>>(mq, mk, mv, mdo, mdk, mdv, macc, prm);
    return cudaGetLastError();
}

}  // namespace fa
