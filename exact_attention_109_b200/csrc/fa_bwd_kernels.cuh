// fa_bwd_kernels.cuh -- backward pass of exact attention for sm_100a.
//
// The gradient of O = softmax(scale Q K^T) V for an upstream dO (the pages
// name gradients and GPT training -- FlashAttention-2 abstract; iplexlaw blog,
// "Tiling preserves the attention calculation": gradient comparisons use
// tolerances -- and print no formula, so this is the textbook derivative):
//     P = exp(scale Q K^T - LSE),   dV = P^T dO,   dP = dO V^T,
//     D_i = rowsum(dO * O)_i,       dS = P * (dP - D),
//     dQ = scale dS K,              dK = scale dS^T Q.
// Three launches:
//   1. fa_bwd_pre_kernel   (HBM-bound) D_i, LSE_i*log2(e), zero fp32 dQ acc.
//   2. fa_bwd_main_kernel  one CTA per (batch*head, 128-row key block j) with
//      K_j, V_j resident in shared memory; it walks the 64-row query blocks
//      (causal: only those at or below the diagonal), recomputes S^T and dP^T
//      on the tensor cores, forms P and dS in registers (one thread per key
//      row), accumulates dV_j and dK_j in TMEM, and adds each block's dQ into
//      the fp32 accumulator with TMA bulk reductions.
//   3. fa_bwd_dq_convert_kernel  dQ = bf16(scale * acc).
// Like the forward pass, nothing N x N is ever written to HBM (the workspace
// is O(N d) per head).
#pragma once

#include <cuda_runtime.h>

#include "sm100_ptx.cuh"

namespace fa {

constexpr int kBwdBM = 64;    // query rows per inner block
constexpr int kBwdBN = 128;   // key rows per CTA

struct BwdWorkspace {
    float* dq_acc;  // [BH, n_pad, d] fp32
    float* lse2;    // [BH, n_pad]    LSE * log2(e); +inf for rows >= N
    float* dvec;    // [BH, n_pad]    rowsum(dO * O); 0 for rows >= N
    int n_pad;      // N rounded up to 128
};

inline size_t bwd_workspace_bytes(long long bh, int N, int d) {
    const long long n_pad = (static_cast<long long>(N) + 127) / 128 * 128;
    return static_cast<size_t>(bh * n_pad * d * 4 + 2 * bh * n_pad * 4);
}

inline BwdWorkspace bwd_workspace_layout(void* base, long long bh, int N, int d) {
    BwdWorkspace ws;
    ws.n_pad = (N + 127) / 128 * 128;
    ws.dq_acc = static_cast<float*>(base);
    ws.lse2 = ws.dq_acc + bh * ws.n_pad * d;
    ws.dvec = ws.lse2 + bh * ws.n_pad;
    return ws;
}

// ------------------------------------------------------------------ 1. pre

// One group of D/8 threads per row; each thread handles 8 columns.
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_pre_kernel(
    const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dO,
    const float* __restrict__ lse, float* __restrict__ dq_acc, float* __restrict__ lse2,
    float* __restrict__ dvec, int N, int n_pad, long long rows_total) {
    constexpr int G = D / 8;
    const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    const long long row = gid / G;
    const int part = static_cast<int>(gid % G);
    const bool valid = row < rows_total;
    const long long bh = row / n_pad;
    const int n = static_cast<int>(row % n_pad);
    float acc = 0.f;
    if (valid && n < N) {
        const size_t off = (static_cast<size_t>(bh) * N + n) * D + part * 8;
        const uint4 a = *reinterpret_cast<const uint4*>(o + off);
        const uint4 b = *reinterpret_cast<const uint4*>(dO + off);
        const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a);
        const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 fa_ = __bfloat1622float2(pa[e]);
            const float2 fb_ = __bfloat1622float2(pb[e]);
            acc = fmaf(fa_.x, fb_.x, acc);
            acc = fmaf(fa_.y, fb_.y, acc);
        }
    }
#pragma unroll
    for (int w = G / 2; w >= 1; w >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, w);
    if (!valid) return;
    if (part == 0) {
        const bool live = n < N;
        dvec[row] = live ? acc : 0.f;
        lse2[row] = live ? lse[static_cast<size_t>(bh) * N + n] * 1.4426950408889634f : INFINITY;
    }
    float4* z = reinterpret_cast<float4*>(dq_acc + row * D + part * 8);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// ------------------------------------------------------------------ 3. dQ

template <int D>
__global__ void __launch_bounds__(256) fa_bwd_dq_convert_kernel(
    const float* __restrict__ dq_acc, __nv_bfloat16* __restrict__ dq, int N, int n_pad,
    long long vec_total, float scale) {
    const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= vec_total) return;  // one thread per 8 output elements
    const long long e = i * 8;
    const long long row = e / D;  // row of the [BH*N, D] output
    const int col = static_cast<int>(e % D);
    const long long bh = row / N;
    const int n = static_cast<int>(row % N);
    const float4* src = reinterpret_cast<const float4*>(
        dq_acc + (static_cast<size_t>(bh) * n_pad + n) * D + col);
    const float4 a = src[0], b = src[1];
    uint4 out;
    out.x = pack_bf16x2(a.x * scale, a.y * scale);
    out.y = pack_bf16x2(a.z * scale, a.w * scale);
    out.z = pack_bf16x2(b.x * scale, b.y * scale);
    out.w = pack_bf16x2(b.z * scale, b.w * scale);
    *reinterpret_cast<uint4*>(dq + e) = out;
}

// ------------------------------------------------------------------ dBias
//
// Causal dBias: the main kernel writes every (query, key) pair of the key
// blocks it visits, from the query block holding the block's first key
// onwards (hidden pairs inside as 0).  The pairs it never visits are those
// of query row q with keys from the next 128-key block on: this kernel
// zeroes exactly those, [128 (floor(q / 128) + 1), N) of every row, with
// 16-byte stores (N % 8 == 0).  One warp per row.
__global__ void __launch_bounds__(256) fa_dbias_zero_upper_kernel(__nv_bfloat16* dbias, int N,
                                                                   long long rows) {
    const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    if (row >= rows) return;
    const int q = static_cast<int>(row % N);
    const int c0 = (q / kBwdBN + 1) * kBwdBN;
    uint4* dst = reinterpret_cast<uint4*>(dbias + row * N);
    for (int c = c0 / 8 + (threadIdx.x & 31); c < N / 8; c += 32) dst[c] = make_uint4(0, 0, 0, 0);
}

// ------------------------------------------------------------------ 2. main

template <int D>
struct BwdTraits {
    static_assert(D == 64 || D == 128, "head dim");
    static constexpr int BN = kBwdBN;
    static constexpr int BM = kBwdBM;
    static constexpr int CH = D / 64;               // 128-byte column chunks
    static constexpr int KV_CHUNK = BN * 128;       // 16 KB
    static constexpr int KV_TILE = BN * D * 2;
    static constexpr int Q_CHUNK = BM * 128;        // 8 KB
    static constexpr int Q_TILE = BM * D * 2;
    static constexpr int NSTAGE = (D == 128) ? 3 : 4;
    static constexpr int STAGE_BYTES = 2 * Q_TILE;  // Q_i then dO_i
    static constexpr int DS_TILE = BN * BM * 2;     // dS^T [128 keys][64 queries] bf16
    static constexpr int DQ_WARP_BYTES = BM * 128;  // fp32 [64 q][32 d] per drain warp
    static constexpr int DQ_WARPS = D / 32;
    static constexpr int K_OFF = 0;
    static constexpr int V_OFF = K_OFF + KV_TILE;   // V follows K directly
    static constexpr int ST_OFF = V_OFF + KV_TILE;
    static constexpr int DS_OFF = ST_OFF + NSTAGE * STAGE_BYTES;
    static constexpr int DQ_OFF = DS_OFF + 2 * DS_TILE;
    static constexpr int VEC_OFF = DQ_OFF + DQ_WARPS * DQ_WARP_BYTES;  // lse2, dvec per stage
    static constexpr int BAR_OFF = VEC_OFF + NSTAGE * 2 * BM * 4;
    // kv, stage_full[NS], stage_empty[NS], sdp_full[2], sdp_loaded[2],
    // pds_ready[2], dq_full[2], dq_drained[2], kv_done, mma_done
    static constexpr int NBAR = 1 + 2 * NSTAGE + 10 + 2;
    static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
    static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;
    // Warps 0-7: two P/dS warpgroups; 8-11: dQ drain; 12: MMA issuer;
    // 13: TMA producer; 14-15 idle.
    static constexpr int NUM_THREADS = 512;
    static constexpr int DRAIN_WARP0 = 8;
    static constexpr int MMA_WARP = 12;
    static constexpr int LOAD_WARP = 13;
    // Register split: P/dS warpgroups grow, dQ drain and MMA/TMA shrink.
    static constexpr uint32_t REG_COMPUTE = 160;
    static constexpr uint32_t REG_DRAIN = 96;
    static constexpr uint32_t REG_CONTROL = 96;
    static constexpr int REG_BUDGET = 128 * (2 * REG_COMPUTE + REG_DRAIN + REG_CONTROL);
    static constexpr uint32_t TMEM_COLS = 512;
    // TMEM columns: buffer b holds S_b at [128b, 128b+64) (later P | dS) and
    // dP_b at [128b+64, 128b+128) (later the dQ^T of the previous block);
    // dV at [256, 256+D), dK at [256+D, 256+2D).
    static constexpr uint32_t DV_COL = 256;
    static constexpr uint32_t DK_COL = 256 + D;
    static constexpr uint32_t IDESC_SDP = idesc_bf16_f32(128, BM, 0, 0);
    static constexpr uint32_t IDESC_ACC = idesc_bf16_f32(128, D, 0, 1);
    static constexpr uint32_t IDESC_DQ = idesc_bf16_f32(128, BM, 1, 1);
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    static_assert(2 * KV_TILE <= NSTAGE * STAGE_BYTES, "dK/dV staging fits the stage ring");
    static_assert(8 * 2 * 4096 <= NSTAGE * STAGE_BYTES, "fp32 dK/dV boxes fit the stage ring");
};

struct BwdParams {
    const float* lse2;
    const float* dvec;
    unsigned int* err;
    int N;
    int n_pad;
    int bh_count;
    int n_kv;        // ceil(N / 128)
    int n_q;         // ceil(N / 64)
    int accum;       // 0: write bf16 dK, dV; 1: add them to fp32 accumulators
    // Additive score bias (null: none): bias [Bb][Hb][N][N] bf16, with
    // Bb = B when bias_batch (else 1) and Hb = H when bias_heads (else 1);
    // dbias (null: not wanted) [B][H][N][N] bf16 receives dS.
    const __nv_bfloat16* bias;
    __nv_bfloat16* dbias;
    int H;
    int bias_batch;
    int bias_heads;
    float scale;
    float scale_log2;
    int strict;      // causal mask without the diagonal: key j visible iff j < i
};

// BIAS: an additive score bias (and optionally its gradient), see BwdParams.
template <int D, bool CAUSAL, bool BIAS = false>
__global__ void __launch_bounds__(512, 1) fa_bwd_main_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
    const __grid_constant__ CUtensorMap tmdK, const __grid_constant__ CUtensorMap tmdV,
    const __grid_constant__ CUtensorMap tmAcc, const BwdParams p) {
    using T = BwdTraits<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::BAR_OFF);
    uint64_t* bar_kv = bars;
    uint64_t* stage_full = bars + 1;
    uint64_t* stage_empty = stage_full + T::NSTAGE;
    uint64_t* sdp_full = stage_empty + T::NSTAGE;
    uint64_t* sdp_loaded = sdp_full + 2;
    uint64_t* pds_ready = sdp_loaded + 2;
    uint64_t* dq_full = pds_ready + 2;
    uint64_t* dq_drained = dq_full + 2;
    uint64_t* kv_done = dq_drained + 2;
    uint64_t* mma_done = kv_done + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + T::MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + T::MISC_OFF + 4);
    float* vec = reinterpret_cast<float*>(smem + T::VEC_OFF);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // Key block j of head bh.  Non-causal: a head's key blocks are adjacent
    // (they share Q and dO in L2).  Causal: key block j walks n_q - 2j query
    // blocks, so the grid takes every head's block 0 first, then every head's
    // block 1, ... (longest first), which keeps a heavy CTA from starting last.
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
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sdp_full[b], 1);
            mbar_init(&sdp_loaded[b], 256);
            mbar_init(&pds_ready[b], 256);
            mbar_init(&dq_full[b], 1);
            mbar_init(&dq_drained[b], 128);
        }
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
    if (warp >= T::MMA_WARP) {
      setmaxnreg_dec<T::REG_CONTROL>();
      if (warp == T::LOAD_WARP) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            bool ok = true;
            mbar_arrive_expect_tx(bar_kv, 2 * T::KV_TILE);
            for (int c = 0; c < T::CH; ++c) {
                tma_load_3d(smem + T::K_OFF + c * T::KV_CHUNK, &tmK, bar_kv, c * 64, j * T::BN, bh);
                tma_load_3d(smem + T::V_OFF + c * T::KV_CHUNK, &tmV, bar_kv, c * 64, j * T::BN, bh);
            }
            int issued = 0;
            for (int k = 0; k < n; ++k) {
                const int s = k % T::NSTAGE;
                const uint32_t par = (k / T::NSTAGE) & 1;
                if (!mbar_wait(&stage_empty[s], par ^ 1u, st)) {
                    ok = false;
                    break;
                }
                const int qrow = (qb0 + k) * T::BM;
                uint8_t* sq = smem + T::ST_OFF + s * T::STAGE_BYTES;
                mbar_arrive_expect_tx(&stage_full[s], T::STAGE_BYTES + 2 * T::BM * 4);
                for (int c = 0; c < T::CH; ++c) {
                    tma_load_3d(sq + c * T::Q_CHUNK, &tmQ, &stage_full[s], c * 64, qrow, bh);
                    tma_load_3d(sq + T::Q_TILE + c * T::Q_CHUNK, &tmdO, &stage_full[s], c * 64,
                                qrow, bh);
                }
                const size_t voff = static_cast<size_t>(bh) * p.n_pad + qrow;
                bulk_load(vec + s * 2 * T::BM, p.lse2 + voff, T::BM * 4, &stage_full[s]);
                bulk_load(vec + s * 2 * T::BM + T::BM, p.dvec + voff, T::BM * 4, &stage_full[s]);
                ++issued;
            }
            if (!ok) {
                for (int k = max(0, issued - T::NSTAGE); k < issued; ++k)
                    mbar_wait_bounded(&stage_full[k % T::NSTAGE], (k / T::NSTAGE) & 1);
                mbar_wait_bounded(bar_kv, 0);
            }
        }
        __syncwarp();
      } else if (warp == T::MMA_WARP) {
        // ------------------------------------------------ MMA issuer
        // This one thread paces the kernel (the P/dS results wait for it),
        // so its hot loop does as little else as possible: the operand
        // descriptors of stage 0, the dS^T buffers and the fixed tiles are
        // built once, barrier addresses stay in registers, and the stage
        // ring advances by adds (no % or / by the stage count).
        if (lane == 0) {
            const uint32_t k_base = smem_u32(smem + T::K_OFF);
            const uint32_t v_base = smem_u32(smem + T::V_OFF);
            const uint32_t st_base = smem_u32(smem + T::ST_OFF);
            const uint32_t ds_base = smem_u32(smem + T::DS_OFF);
            // S^T_b = K Q^T and dP^T_b = V dO^T: M=128 keys, N=64 queries, K=D.
            // Base descriptors of the fixed tiles; K steps add byte offsets.
            const uint64_t dk0 = sdesc_sw128(k_base, 16, 1024);
            const uint64_t dv0 = sdesc_sw128(v_base, 16, 1024);
            const uint64_t dkt0 = sdesc_sw128(k_base, T::KV_CHUNK, 1024);
            // Stage 0's Q and dO, K-major (S^T, dP^T) and MN-major (dV, dK);
            // stage s adds s * STAGE_BYTES.
            const uint64_t sq_k = sdesc_sw128(st_base, 16, 1024);
            const uint64_t sdo_k = sdesc_sw128(st_base + T::Q_TILE, 16, 1024);
            const uint64_t sq_mn = sdesc_sw128(st_base, T::Q_CHUNK, 1024);
            const uint64_t sdo_mn = sdesc_sw128(st_base + T::Q_TILE, T::Q_CHUNK, 1024);
            const uint64_t dds_b0 = sdesc_sw128(ds_base, T::DS_TILE, 1024);  // dS^T buffer 0
            const uint32_t sfull_a = smem_u32(stage_full), sempty_a = smem_u32(stage_empty);
            const uint32_t sdpf_a = smem_u32(sdp_full), sdpl_a = smem_u32(sdp_loaded);
            const uint32_t pds_a = smem_u32(pds_ready), dqf_a = smem_u32(dq_full);
            const uint32_t dqd_a = smem_u32(dq_drained);
            auto mma_sdp = [&](uint32_t soff, int b) {  // soff: the stage's byte offset
                const uint64_t dq0 = sdesc_add(sq_k, soff);
                const uint64_t ddo0 = sdesc_add(sdo_k, soff);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t offk = (kk >> 2) * T::KV_CHUNK + (kk & 3) * 32;
                    const uint32_t offq = (kk >> 2) * T::Q_CHUNK + (kk & 3) * 32;
                    if (kk == 0)
                        umma_ss_c<false>(tmem + 128u * b, dk0, dq0, T::IDESC_SDP);
                    else
                        umma_ss_c<true>(tmem + 128u * b, sdesc_add(dk0, offk),
                                        sdesc_add(dq0, offq), T::IDESC_SDP);
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t offk = (kk >> 2) * T::KV_CHUNK + (kk & 3) * 32;
                    const uint32_t offq = (kk >> 2) * T::Q_CHUNK + (kk & 3) * 32;
                    if (kk == 0)
                        umma_ss_c<false>(tmem + 128u * b + 64u, dv0, ddo0, T::IDESC_SDP);
                    else
                        umma_ss_c<true>(tmem + 128u * b + 64u, sdesc_add(dv0, offk),
                                        sdesc_add(ddo0, offq), T::IDESC_SDP);
                }
            };
            // dV += P^T dO and dK += dS^T Q: M=128 keys, N=D, K=64 queries;
            // A (P^T or dS^T) from TMEM, B (dO or Q) MN-major from the stage.
            auto mma_dkdv = [&](uint32_t soff, bool first, int b) {
                const uint64_t bq0 = sdesc_add(sq_mn, soff);
                const uint64_t bdo0 = sdesc_add(sdo_mn, soff);
#pragma unroll
                for (int kk = 0; kk < T::BM / 16; ++kk) {
                    const uint32_t a_col = 128u * b + 32u * (kk >> 1) + 8u * (kk & 1);
                    if (kk == 0) {  // the first query block overwrites, later ones accumulate
                        umma_ts(tmem + T::DV_COL, tmem + a_col, bdo0, T::IDESC_ACC, first ? 0u : 1u);
                        umma_ts(tmem + T::DK_COL, tmem + a_col + 16u, bq0, T::IDESC_ACC,
                                first ? 0u : 1u);
                    } else {
                        umma_ts_c<true>(tmem + T::DV_COL, tmem + a_col, sdesc_add(bdo0, kk * 2048),
                                        T::IDESC_ACC);
                        umma_ts_c<true>(tmem + T::DK_COL, tmem + a_col + 16u,
                                        sdesc_add(bq0, kk * 2048), T::IDESC_ACC);
                    }
                }
            };
            // dQ^T = K^T dS^T: M=128 (head dim; rows >= D unused), N=64
            // queries, K=128 keys; both operands MN-major in shared memory.
            auto mma_dq = [&](int bs, int b1) {  // bs: the dS^T buffer
                const uint64_t dds0 = sdesc_add(dds_b0, bs * T::DS_TILE);
#pragma unroll
                for (int kk = 0; kk < T::BN / 16; ++kk) {
                    if (kk == 0)
                        umma_ss_c<false>(tmem + 128u * b1 + 64u, dkt0, dds0, T::IDESC_DQ);
                    else
                        umma_ss_c<true>(tmem + 128u * b1 + 64u, sdesc_add(dkt0, kk * 2048),
                                        sdesc_add(dds0, kk * 2048), T::IDESC_DQ);
                }
            };
            bool ok = mbar_wait(bar_kv, 0, st);
            for (int k = 0; k < 2 && k < n && ok; ++k) {  // stages 0 and 1, phase 0
                ok = mbar_wait_s(sfull_a + 8u * k, 0, st);
                if (!ok) break;
                tc_fence_after();
                mma_sdp(static_cast<uint32_t>(k) * T::STAGE_BYTES, k);
                umma_commit_s(sdpf_a + 8u * k);
            }
            // Stage slot of block k (s0) and of block k+2 (s2, with its phase
            // parity p2), advanced by one slot per block.
            uint32_t s0 = 0, s2 = 2u % T::NSTAGE, p2 = (2u / T::NSTAGE) & 1u;
            for (int k = 0; k < n && ok; ++k) {
                const int b = k & 1, b1 = b ^ 1;
                if (!(ok = mbar_wait_s(pds_a + 8u * b, (k >> 1) & 1, st))) break;
                tc_fence_after();
                mma_dkdv(s0 * T::STAGE_BYTES, k == 0, b);
                if (k + 1 < n)
                    ok = mbar_wait_s(sdpl_a + 8u * b1, ((k + 1) >> 1) & 1, st);
                else if (k >= 2)
                    ok = mbar_wait_s(dqd_a + 8u * b1, ((k - 2) >> 1) & 1, st);
                if (!ok) break;
                tc_fence_after();
                mma_dq(b, b1);
                umma_commit_s(dqf_a + 8u * b1);
                umma_commit_s(sempty_a + 8u * s0);
                if (k + 2 < n) {
                    ok = mbar_wait_s(sfull_a + 8u * s2, p2, st);
                    if (ok && k >= 1) ok = mbar_wait_s(dqd_a + 8u * b, ((k - 1) >> 1) & 1, st);
                    if (!ok) break;
                    tc_fence_after();
                    mma_sdp(s2 * T::STAGE_BYTES, b);
                    // This commit completes only after dQ^T(k) above has read
                    // dS^T buffer k & 1, which block k+2's P/dS warps rewrite
                    // once they see it: keep S/dP(k+2) after dQ^T(k).
                    umma_commit_s(sdpf_a + 8u * b);
                }
                if (++s0 == T::NSTAGE) s0 = 0;
                if (++s2 == T::NSTAGE) {
                    s2 = 0;
                    p2 ^= 1u;
                }
            }
            if (ok) umma_commit(kv_done);
            umma_commit(mma_done);
            mbar_wait_bounded(mma_done, 0);
        }
        __syncwarp();
      }
    } else if (warp < T::DRAIN_WARP0) {
        // ------------------------------------------------ P / dS (one thread per key row)
        // Two warpgroups: warpgroup g handles query columns [32g, 32g+32) of
        // every key row and rewrites only its own 32 S columns (P, then dS).
        setmaxnreg_inc<T::REG_COMPUTE>();
        const int g = warp >> 2;
        const int lg = warp & 3;
        const int r = lg * 32 + lane;
        const int kv_row = j * T::BN + r;
        // Key rows past N (zero-filled K, V): P = 0, so that a score of 0
        // against a very negative LSE cannot overflow into dS.
        const bool row_live = kv_row < N;
        const uint32_t lane_off = static_cast<uint32_t>(lg * 32) << 16;
        const float sl2 = p.scale_log2;
        // Bias and its gradient are read and written straight from / to HBM:
        // for a fixed query row the 32 lanes of a warp touch 32 consecutive
        // keys (64 contiguous bytes) per instruction.
        const __nv_bfloat16* bias_base = nullptr;
        if (BIAS) {
            const int bb = bh / p.H, hh = bh % p.H;
            const long long bz = static_cast<long long>(p.bias_batch ? bb : 0) *
                                     (p.bias_heads ? p.H : 1) + (p.bias_heads ? hh : 0);
            bias_base = p.bias + bz * N * N;
        }
        __nv_bfloat16* dbias_base =
            BIAS && p.dbias ? p.dbias + static_cast<long long>(bh) * N * N : nullptr;
        // Bias b[q][key] of a block's 32 query columns.  The loads run one
        // block ahead: block k+1's are issued at the top of block k (raw
        // 16-bit values, one register each) and packed at its end, so an HBM
        // round trip never stalls a block.
        unsigned short braw[32];
        uint32_t bpk[16];
        auto bias_load = [&](int kk) {
            const int q0 = (qb0 + kk) * T::BM + 32 * g;
            const unsigned short* bp = reinterpret_cast<const unsigned short*>(bias_base) +
                                       static_cast<long long>(q0) * N + kv_row;
#pragma unroll
            for (int e = 0; e < 32; ++e)
                braw[e] = (kv_row < N && q0 + e < N) ? __ldg(bp + static_cast<long long>(e) * N)
                                                     : static_cast<unsigned short>(0);
        };
        auto bias_pack = [&]() {
#pragma unroll
            for (int e = 0; e < 16; ++e)
                bpk[e] = static_cast<uint32_t>(braw[2 * e]) |
                         (static_cast<uint32_t>(braw[2 * e + 1]) << 16);
        };
        if constexpr (BIAS) {
            bias_load(0);
            bias_pack();
        }
        bool ok = true;
        for (int k = 0; k < n; ++k) {
            const int b = k & 1;
            if constexpr (BIAS) {
                if (k + 1 < n) bias_load(k + 1);
            }
            ok = __all_sync(0xffffffffu, mbar_wait(&sdp_full[b], (k >> 1) & 1, st));
            if (!ok) break;
            tc_fence_after();
            const uint32_t s_tm = tmem + lane_off + 128u * b + 32u * g;
            uint32_t sv[32], dp[32];
            tmem_ld32(s_tm, sv);
            tmem_ld32(s_tm + 64u, dp);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(&sdp_loaded[b]);

            const float4* l4 = reinterpret_cast<const float4*>(vec + (k % T::NSTAGE) * 2 * T::BM +
                                                               32 * g);
            const float4* d4 = l4 + T::BM / 4;
            const int qrow0 = (qb0 + k) * T::BM + 32 * g;
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
                for (int h = 0; h < 4; ++h) {
                    const int e = 4 * e4 + h;
                    float arg = -lsv[h];
                    if constexpr (BIAS) {
                        const uint32_t w = bpk[e >> 1];
                        const float bv = __uint_as_float((e & 1) ? (w & 0xffff0000u) : (w << 16));
                        arg = fmaf(bv, 1.4426950408889634f, arg);
                    }
                    float x = ex2_approx(fmaf(__uint_as_float(sv[e]), sl2, arg));
                    if (!row_live || (CAUSAL && e < masked)) x = 0.f;
                    pr[h] = x;
                    ds[h] = x * (__uint_as_float(dp[e]) - dsv_[h]);
                }
                pk[2 * e4] = pack_bf16x2(pr[0], pr[1]);
                pk[2 * e4 + 1] = pack_bf16x2(pr[2], pr[3]);
                dk[2 * e4] = pack_bf16x2(ds[0], ds[1]);
                dk[2 * e4 + 1] = pack_bf16x2(ds[2], ds[3]);
            }
            if (BIAS && dbias_base && kv_row < N) {
                // dBias = dS, rounded to bf16 as for the dQ and dK MMAs
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    if (qrow0 + e < N)
                        *reinterpret_cast<unsigned short*>(
                            dbias_base + static_cast<long long>(qrow0 + e) * N + kv_row) =
                            static_cast<unsigned short>((e & 1) ? (dk[e >> 1] >> 16)
                                                                : (dk[e >> 1] & 0xffffu));
            }
            // P^T then dS^T over this warpgroup's own S columns (A operands of
            // the dV and dK MMAs).
            tmem_st16(s_tm, pk);
            tmem_st16(s_tm + 16u, dk);
            // dS^T half-row to shared memory (B operand of dQ^T), 128-byte swizzle.
            uint8_t* dsrow = smem + T::DS_OFF + (k & 1) * T::DS_TILE;
#pragma unroll
            for (int u = 0; u < 4; ++u)
                *reinterpret_cast<uint4*>(dsrow + sw128_offset(r, 4 * g + u)) =
                    make_uint4(dk[4 * u], dk[4 * u + 1], dk[4 * u + 2], dk[4 * u + 3]);
            fence_proxy_async_smem();
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&pds_ready[b]);
            if constexpr (BIAS) {
                if (k + 1 < n) bias_pack();
            }
        }
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(kv_done, 0, st));
        if (ok && p.accum) {
            // Accumulating: warpgroup 0 adds dV, warpgroup 1 adds scale*dK
            // to fp32 [B*H][N][D] buffers with TMA bulk reduce-adds of
            // [32 rows][32 head dims] boxes (128-byte swizzle), staged two
            // boxes per warp in the stage ring, which no MMA reads any more.
            tc_fence_after();
            const uint32_t col0 = g ? T::DK_COL : T::DV_COL;
            const float mul = g ? p.scale : 1.0f;
            uint8_t* stage = smem + T::ST_OFF + (g * 4 + lg) * 2 * 4096;
            const int wrow0 = j * T::BN + lg * 32;
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                uint32_t a[32];
                tmem_ld32(tmem + lane_off + col0 + 32u * c, a);
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
                    tma_reduce_add_3d(g ? &tmdK : &tmdV, box, 32 * c, wrow0, bh);
                    bulk_commit_group();
                }
            }
            if (lane == 0 && wrow0 < N) bulk_wait_group0();
        } else if (ok) {
            // Warpgroup 0 writes dV, warpgroup 1 writes scale*dK: bf16, staged
            // (128-byte swizzle) in the stage ring, which no MMA reads any
            // more; TMA-stored 32 rows per warp.
            tc_fence_after();
            const uint32_t col0 = g ? T::DK_COL : T::DV_COL;
            const float mul = g ? p.scale : 1.0f;
            uint8_t* stage = smem + T::ST_OFF + g * T::KV_TILE + lg * 32 * 128;
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                uint32_t a[32];
                tmem_ld32(tmem + lane_off + col0 + 32u * c, a);
                tmem_ld_wait();
                uint8_t* chunk = stage + (c >> 1) * T::KV_CHUNK;
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
                    *reinterpret_cast<uint4*>(chunk + sw128_offset(lane, (c & 1) * 4 + u)) = v;
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            const int wrow0 = j * T::BN + lg * 32;
            if (lane == 0 && wrow0 < N) {
                for (int c = 0; c < T::CH; ++c)
                    tma_store_3d(g ? &tmdK : &tmdV, stage + c * T::KV_CHUNK, c * 64, wrow0, bh);
                bulk_commit_group();
                bulk_wait_group_read0();
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ dQ drain (warps 8-11)
        setmaxnreg_dec<T::REG_DRAIN>();
        const int lg = warp - T::DRAIN_WARP0;  // TMEM lanes [32 lg, 32 lg + 32) = head dims
        const uint32_t lane_off = static_cast<uint32_t>(lg * 32) << 16;
        const bool live = lg * 32 < D;         // head dims >= D are padding
        uint8_t* buf = smem + T::DQ_OFF + (live ? lg : 0) * T::DQ_WARP_BYTES;
        for (int k = 0; k < n; ++k) {
            const int b1 = (k + 1) & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&dq_full[b1], (k >> 1) & 1, st))) break;
            tc_fence_after();
            uint32_t a[2][32];
            if (live) {
                tmem_ld32(tmem + lane_off + 128u * b1 + 64u, a[0]);
                tmem_ld32(tmem + lane_off + 128u * b1 + 96u, a[1]);
                tmem_ld_wait();
            }
            tc_fence_before();
            mbar_arrive(&dq_drained[b1]);
            if (live) {
                if (lane == 0) bulk_wait_group_read0();  // previous reduce has read buf
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
        }
        if (live && lane == 0) bulk_wait_group0();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == T::MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem, T::TMEM_COLS);
    }
}

// ------------------------------------------------------------------ launch

// Stage 1: D, log2-scaled LSE and the zeroed dQ accumulator.
template <int D>
cudaError_t launch_bwd_pre(const void* o, const float* lse, const void* dO, int bh, int N,
                           const BwdWorkspace& ws, cudaStream_t s) {
    const long long rows = static_cast<long long>(bh) * ws.n_pad;
    const long long threads = rows * (D / 8);
    fa_bwd_pre_kernel<D><<<static_cast<unsigned>((threads + 255) / 256), 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dO), lse,
        ws.dq_acc, ws.lse2, ws.dvec, N, ws.n_pad, rows);
    return cudaGetLastError();
}

// Stage 2: dK, dV and the fp32 dQ accumulation (needs stage 1's workspace).
template <int D, bool CAUSAL, bool BIAS = false>
cudaError_t launch_bwd_main(int bh, int N, float scale, const BwdWorkspace& ws,
                            const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                            const CUtensorMap& mdo, const CUtensorMap& mdk,
                            const CUtensorMap& mdv, const CUtensorMap& macc, unsigned int* err,
                            cudaStream_t s, int accum = 0, const void* bias = nullptr,
                            void* dbias = nullptr, int H = 1, int bias_batch = 0,
                            int bias_heads = 0, int strict = 0) {
    using T = BwdTraits<D>;
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
    prm.bias = static_cast<const __nv_bfloat16*>(bias);
    prm.dbias = static_cast<__nv_bfloat16*>(dbias);
    prm.H = H;
    prm.bias_batch = bias_batch;
    prm.bias_heads = bias_heads;
    prm.scale = scale;
    prm.scale_log2 = scale * 1.4426950408889634f;
    prm.strict = strict;
    const long long grid = static_cast<long long>(bh) * prm.n_kv;
    fa_bwd_main_kernel<D, CAUSAL, BIAS><<<static_cast<unsigned>(grid), T::NUM_THREADS,
                                          T::SMEM_BYTES, s>>>(
        mq, mk, mv, mdo, mdk, mdv, macc, prm);
    return cudaGetLastError();
}

// Stage 3: dQ = bf16(scale * accumulator).
template <int D>
cudaError_t launch_bwd_convert(void* dq, int bh, int N, float scale, const BwdWorkspace& ws,
                               cudaStream_t s) {
    const long long vecs = static_cast<long long>(bh) * N * D / 8;
    fa_bwd_dq_convert_kernel<D><<<static_cast<unsigned>((vecs + 255) / 256), 256, 0, s>>>(
        ws.dq_acc, static_cast<__nv_bfloat16*>(dq), N, ws.n_pad, vecs, scale);
    return cudaGetLastError();
}

}  // namespace fa
