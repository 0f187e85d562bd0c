// fa_decode_kernel.cuh -- split-KV forward attention for decoding: a few
// query rows (N_q, typically 1) against a long cache of N_k keys.
//
// iplexlaw blog "FlashAttention-2 GPU work partitioning", section "What the
// paper measures": prefill and token-by-token decoding have different
// bottlenecks and are measured apart.  With N_q rows each cached key row is
// used for only 4 * N_q * d FLOPs, so decoding is bound by reading K and V
// from HBM, not by the tensor cores: these kernels stream K/V through shared
// memory with bulk asynchronous copies and do the arithmetic on the fp32
// CUDA cores.  To keep every SM streaming when B*H is small, the key range of
// one head is cut into splits, each CTA reduces one split to a partial
// (O_s / l_s, log2 l_s + m_s), and a second kernel merges the partials with
// the log-sum-exp rule -- the same rescaling that the online softmax
// ("Tiling preserves the attention calculation") applies block by block.
//
// Causal masking for N_q != N_k aligns the query rows with the LAST N_q keys:
// query i (0-based) sees key j iff j <= i + N_k - N_q, which reduces to the
// j <= i of the square case when N_q = N_k.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "sm100_ptx.cuh"

namespace fa {

struct DecodeParams {
    const __nv_bfloat16* q;  // [BH][Nq][D]
    const __nv_bfloat16* k;  // [BH][kv_rows][D], first Nk rows used
    const __nv_bfloat16* v;
    __nv_bfloat16* o;  // [BH][Nq][D]       written when n_splits == 1
    float* lse;        // [BH][Nq] (natural log), written when n_splits == 1
    float* part_o;     // [BH][Nq][n_splits][D]  O_s / l_s     (n_splits > 1)
    float* part_lse;   // [BH][Nq][n_splits]     m_s + log2 l_s (n_splits > 1)
    unsigned int* err;
    long long kv_rows;  // rows per head in the k and v buffers (>= Nk)
    int Nq, Nk;
    int n_qgroups;  // ceil(Nq / QG)
    int n_splits;   // key splits per (head, query group)
    int chunk;      // keys per split, a multiple of BK
    int causal;
    float scale_log2;  // scale * log2(e)
};

template <int D>
struct DecTraits {
    static constexpr int G = 8;            // lanes that share one key row
    static constexpr int E = D / G;        // head-dim elements per lane: 8 or 16
    static constexpr int NCW = 4;          // consumer warps
    static constexpr int NGRP = NCW * 32 / G;  // key groups per CTA (16)
    static constexpr int KPG = 4;          // keys per group per block
    static constexpr int BK = NGRP * KPG;  // keys per pipeline stage (64)
    static constexpr int NSTAGE = D == 128 ? 3 : 4;
    static constexpr int TILE_BYTES = BK * D * 2;         // one of K, V
    static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
    static constexpr int THREADS = (NCW + 1) * 32;        // + one producer warp
    static constexpr int BAR_OFF = NSTAGE * STAGE_BYTES;
    static constexpr int SMEM_BYTES = BAR_OFF + 1024;
    // Resident CTAs per SM the register budget is fitted to (shared memory
    // allows 2 at D = 128 and 3 at D = 64).
    static constexpr int MIN_CTAS = D == 128 ? 2 : 3;
    static_assert(E == 8 || E == 16, "head dim must be 64 or 128");
};

// Keys are cut into splits of at least this many, so the partial-result
// workspace is bounded by ceil(Nk / kDecodeMinChunk) splits per row.
constexpr int kDecodeMinChunk = 256;

// Eight bf16 values (one 16-byte load) as four fp32 pairs.
__device__ __forceinline__ void unpack8(const uint4& w, uint64_t (&f)[4]) {
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
        f[i] = f2_pack(__uint_as_float(u[i] << 16), __uint_as_float(u[i] & 0xffff0000u));
}

// Element offsets (within a row of D) of the E elements that lane c of a key
// group owns: [8c, 8c + 8) and, for D = 128, [64 + 8c, 64 + 8c + 8).  Each
// 16-byte load of one group then covers 128 contiguous bytes of one row.
template <int D>
__device__ __forceinline__ int dec_col(int c, int half) {
    return 8 * c + 64 * half;
}

// Grid: one CTA per (head, key split, query group), query groups fastest so
// that CTAs reading the same keys run together and share them through L2.
template <int D, int QG>
__global__ void __launch_bounds__(DecTraits<D>::THREADS, DecTraits<D>::MIN_CTAS)
    fa_decode_kernel(const DecodeParams p) {
    using T = DecTraits<D>;
    constexpr int NH = T::E / 8;  // 16-byte loads per row per lane (1 or 2)
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + T::BAR_OFF);
    uint64_t* empty = full + T::NSTAGE;
    float* red_ml = reinterpret_cast<float*>(empty + T::NSTAGE);  // [NGRP][QG][2]
    volatile int* abort_flag = reinterpret_cast<volatile int*>(red_ml + T::NGRP * QG * 2);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // The merge kernel may be scheduled now; it waits for this grid to end.
    grid_launch_dependents();
    int idx = blockIdx.x;
    const int qg = idx % p.n_qgroups;
    idx /= p.n_qgroups;
    const int split = idx % p.n_splits;
    const long long bh = idx / p.n_splits;
    const int i0 = qg * QG;
    const int i_last = min(i0 + QG, p.Nq) - 1;
    const int kvis = p.causal ? min(p.Nk, i_last + p.Nk - p.Nq + 1) : p.Nk;
    const int kbeg = split * p.chunk;
    const int kend = min(kbeg + p.chunk, kvis);
    const int nblk = kend > kbeg ? (kend - kbeg + T::BK - 1) / T::BK : 0;

    if (nblk == 0) {
        // Nothing visible in this split (causal rows of an early query
        // group): an empty partial, weight zero in the merge.  (With one
        // split every row sees key 0, so this only happens to partials.)
        if (p.n_splits == 1) return;
        for (int t = threadIdx.x; t < QG * D; t += T::THREADS) {
            const int r = t / D, e = t % D, row = i0 + r;
            if (row >= p.Nq) continue;
            const long long pr = (bh * p.Nq + row) * p.n_splits + split;
            p.part_o[pr * D + e] = 0.f;
            if (e == 0) p.part_lse[pr] = -INFINITY;
        }
        return;
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < T::NSTAGE; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], T::NCW);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    const AbortState st{reinterpret_cast<volatile int*>(abort_flag), p.err};

    if (warp == T::NCW) {
        // ------------------------------------------------ producer
        if (lane == 0) {
            const __nv_bfloat16* kh = p.k + bh * p.kv_rows * D;
            const __nv_bfloat16* vh = p.v + bh * p.kv_rows * D;
            int issued = 0;
            for (int b = 0; b < nblk; ++b) {
                const int s = b % T::NSTAGE;
                if (b >= T::NSTAGE && !mbar_wait(&empty[s], ((b / T::NSTAGE) - 1) & 1, st))
                    break;
                const int j0 = kbeg + b * T::BK;
                const uint32_t bytes = static_cast<uint32_t>(min(T::BK, kend - j0)) * D * 2;
                uint8_t* kt = smem + s * T::STAGE_BYTES;
                mbar_arrive_expect_tx(&full[s], 2 * bytes);
                bulk_load(kt, kh + static_cast<long long>(j0) * D, bytes, &full[s]);
                bulk_load(kt + T::TILE_BYTES, vh + static_cast<long long>(j0) * D, bytes,
                          &full[s]);
                issued = b + 1;
            }
            // Do not leave with copies in flight: wait (bounded) for the last
            // stages issued; earlier ones were consumed before being reused.
            for (int b = max(0, issued - T::NSTAGE); b < issued; ++b)
                mbar_wait_bounded(&full[b % T::NSTAGE], (b / T::NSTAGE) & 1);
        }
        return;
    }

    // ---------------------------------------------------- consumers
    const int g = warp * (32 / T::G) + (lane >> 3);  // key group
    const int c = lane & 7;                           // lane within the group
    const int hi4 = (c >> 2) & 1, hi2 = (c >> 1) & 1;
    const int t_own = 2 * hi4 + hi2;  // key slot this lane ends up holding

    // Query rows, pre-multiplied by scale * log2(e) so that scores come out
    // in the base-2 domain of the softmax below.
    uint64_t qf[QG][T::E / 2];
    int lim[QG];
#pragma unroll
    for (int r = 0; r < QG; ++r) {
        const int row = min(i0 + r, p.Nq - 1);
        lim[r] = p.causal ? row + p.Nk - p.Nq : 0x7fffffff;
        const __nv_bfloat16* qr = p.q + (bh * p.Nq + row) * D;
#pragma unroll
        for (int h = 0; h < NH; ++h) {
            uint64_t f[4];
            unpack8(*reinterpret_cast<const uint4*>(qr + dec_col<D>(c, h)), f);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float a, b2;
                f2_unpack(f[i], a, b2);
                qf[r][4 * h + i] = f2_pack(a * p.scale_log2, b2 * p.scale_log2);
            }
        }
    }

    float m[QG], l[QG];
    uint64_t o[QG][T::E / 2];
#pragma unroll
    for (int r = 0; r < QG; ++r) {
        m[r] = -INFINITY;
        l[r] = 0.f;
#pragma unroll
        for (int e = 0; e < T::E / 2; ++e) o[r][e] = 0ull;
    }

    for (int b = 0; b < nblk; ++b) {
        const int s = b % T::NSTAGE;
        if (!mbar_wait(&full[s], (b / T::NSTAGE) & 1, st)) break;
        const uint8_t* kt = smem + s * T::STAGE_BYTES;
        const uint8_t* vt = kt + T::TILE_BYTES;
        const int j0 = kbeg + b * T::BK;
        const int nk = min(T::BK, kend - j0);

        // S = Q K^T: lane c forms partial dot products over its E columns for
        // the group's KPG keys (block rows t * NGRP + g).
        float acc[QG][T::KPG];
#pragma unroll
        for (int t = 0; t < T::KPG; ++t) {
            const uint8_t* kr = kt + (t * T::NGRP + g) * (D * 2);
            uint64_t kf[T::E / 2];
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                uint64_t f[4];
                unpack8(*reinterpret_cast<const uint4*>(kr + 2 * dec_col<D>(c, h)), f);
#pragma unroll
                for (int i = 0; i < 4; ++i) kf[4 * h + i] = f[i];
            }
#pragma unroll
            for (int r = 0; r < QG; ++r) {
                uint64_t a2 = ffma2(qf[r][0], kf[0], 0ull);
#pragma unroll
                for (int e = 1; e < T::E / 2; ++e) a2 = ffma2(qf[r][e], kf[e], a2);
                float lo, hi;
                f2_unpack(a2, lo, hi);
                acc[r][t] = lo + hi;
            }
        }

        // Sum the partial dot products over the group's 8 lanes, transposing
        // as we go: after the xor-4 and xor-2 steps each lane holds one key's
        // sum over half, then all, of the lanes, so no lane sums a value that
        // another lane also sums.  Lane c ends with key slot t_own.
        float sc[QG];
#pragma unroll
        for (int r = 0; r < QG; ++r) {
            float b2[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const float send = hi4 ? acc[r][u] : acc[r][2 + u];
                const float keep = hi4 ? acc[r][2 + u] : acc[r][u];
                b2[u] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
            }
            const float send = hi2 ? b2[0] : b2[1];
            const float keep = hi2 ? b2[1] : b2[0];
            const float cc = keep + __shfl_xor_sync(0xffffffffu, send, 2);
            sc[r] = cc + __shfl_xor_sync(0xffffffffu, cc, 1);
        }

        // Mask, then the online-softmax update with deferred rescaling: the
        // running max moves only when a block's max exceeds it by more than
        // 8 (weights stay <= 2^8 in fp32), which skips most rescales of O.
        const int jb = t_own * T::NGRP + g;  // block row of this lane's key
        const bool in_blk = jb < nk;
        float pw[QG];
#pragma unroll
        for (int r = 0; r < QG; ++r) {
            const float sv = (in_blk && j0 + jb <= lim[r]) ? sc[r] : -INFINITY;
            float bm = fmaxf(sv, __shfl_xor_sync(0xffffffffu, sv, 2));
            bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 4));
            if (bm > m[r] + 8.f) {
                const float alpha = ex2_approx(m[r] - bm);  // 0 while m = -inf
                const uint64_t a2 = f2_pack(alpha, alpha);
                l[r] *= alpha;
#pragma unroll
                for (int e = 0; e < T::E / 2; ++e) o[r][e] = ffma2(o[r][e], a2, 0ull);
                m[r] = bm;
            }
            // m[r] is finite whenever sv is (a finite score raises it above).
            pw[r] = sv == -INFINITY ? 0.f : ex2_approx(sv - m[r]);
            l[r] += pw[r];
        }

        // O += P V: each key's weight is broadcast from the lane that holds
        // it; rows past the end of the block hold stale data and are skipped.
        float pt[T::KPG][QG];
#pragma unroll
        for (int t = 0; t < T::KPG; ++t) {
            const int src = (lane & ~7) | ((t >> 1) << 2) | ((t & 1) << 1);
#pragma unroll
            for (int r = 0; r < QG; ++r) pt[t][r] = __shfl_sync(0xffffffffu, pw[r], src);
        }
#pragma unroll
        for (int t = 0; t < T::KPG; ++t) {
            if (t * T::NGRP + g < nk) {
                const uint8_t* vr = vt + (t * T::NGRP + g) * (D * 2);
                uint64_t vf[T::E / 2];
#pragma unroll
                for (int h = 0; h < NH; ++h) {
                    uint64_t f[4];
                    unpack8(*reinterpret_cast<const uint4*>(vr + 2 * dec_col<D>(c, h)), f);
#pragma unroll
                    for (int i = 0; i < 4; ++i) vf[4 * h + i] = f[i];
                }
#pragma unroll
                for (int r = 0; r < QG; ++r) {
                    const uint64_t p2 = f2_pack(pt[t][r], pt[t][r]);
#pragma unroll
                    for (int e = 0; e < T::E / 2; ++e) o[r][e] = ffma2(p2, vf[e], o[r][e]);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
    }

    // Per-group row sums: lanes c, c^2, c^4, c^6 hold the four distinct keys
    // (c^1 duplicates c).
#pragma unroll
    for (int r = 0; r < QG; ++r) {
        l[r] += __shfl_xor_sync(0xffffffffu, l[r], 2);
        l[r] += __shfl_xor_sync(0xffffffffu, l[r], 4);
    }

    // Merge the NGRP groups' (m, l, O) through shared memory, in the stage
    // buffers: every copy has landed (each stage was waited on), and the
    // barrier below holds the writes until no consumer reads a stage.
    float* ored = reinterpret_cast<float*>(smem);  // [NGRP][QG][D]
    static_assert(T::NGRP * QG * D * 4 <= T::BAR_OFF, "merge buffer exceeds the stages");
    named_bar_sync(1, T::NCW * 32);
#pragma unroll
    for (int r = 0; r < QG; ++r) {
        if (c == 0) {
            red_ml[(g * QG + r) * 2 + 0] = m[r];
            red_ml[(g * QG + r) * 2 + 1] = l[r];
        }
        float* dst = ored + (g * QG + r) * D;
#pragma unroll
        for (int h = 0; h < NH; ++h) {
            float w[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) f2_unpack(o[r][4 * h + i], w[2 * i], w[2 * i + 1]);
            float4* d4 = reinterpret_cast<float4*>(dst + dec_col<D>(c, h));
            d4[0] = make_float4(w[0], w[1], w[2], w[3]);
            d4[1] = make_float4(w[4], w[5], w[6], w[7]);
        }
    }
    named_bar_sync(1, T::NCW * 32);

    for (int t = threadIdx.x; t < QG * (D / 4); t += T::NCW * 32) {
        const int r = t / (D / 4), e4 = (t % (D / 4)) * 4;
        const int row = i0 + r;
        if (row >= p.Nq) continue;
        float M = -INFINITY;
#pragma unroll
        for (int gg = 0; gg < T::NGRP; ++gg) M = fmaxf(M, red_ml[(gg * QG + r) * 2]);
        float L = 0.f;
        float4 acc4 = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int gg = 0; gg < T::NGRP; ++gg) {
            const float mg = red_ml[(gg * QG + r) * 2];
            const float w = mg == -INFINITY ? 0.f : ex2_approx(mg - M);
            L += w * red_ml[(gg * QG + r) * 2 + 1];
            const float4 x = *reinterpret_cast<const float4*>(ored + (gg * QG + r) * D + e4);
            acc4.x += w * x.x;
            acc4.y += w * x.y;
            acc4.z += w * x.z;
            acc4.w += w * x.w;
        }
        const long long orow = bh * p.Nq + row;
        if (p.n_splits == 1) {
            const float inv = 1.f / L;  // L > 0: row `row` sees key 0
            uint2 packed;
            packed.x = pack_bf16x2(acc4.x * inv, acc4.y * inv);
            packed.y = pack_bf16x2(acc4.z * inv, acc4.w * inv);
            *reinterpret_cast<uint2*>(p.o + orow * D + e4) = packed;
            if (e4 == 0) p.lse[orow] = (M + __log2f(L)) * 0.6931471805599453f;
        } else {
            const long long pr = orow * p.n_splits + split;
            const float inv = L > 0.f ? 1.f / L : 0.f;
            *reinterpret_cast<float4*>(p.part_o + pr * D + e4) =
                make_float4(acc4.x * inv, acc4.y * inv, acc4.z * inv, acc4.w * inv);
            if (e4 == 0) p.part_lse[pr] = L > 0.f ? M + __log2f(L) : -INFINITY;
        }
    }
}

// Merges the n_splits partials of every output row: with w_s = 2^(lse_s - M),
// O = sum_s w_s O_s / sum_s w_s and LSE = (M + log2 sum_s w_s) * ln 2.
// One warp per row; lane l owns D/32 consecutive columns.
template <int D>
__global__ void __launch_bounds__(128) fa_decode_combine_kernel(const float* __restrict__ part_o,
                                                                const float* __restrict__ part_lse,
                                                                __nv_bfloat16* o, float* lse,
                                                                long long rows, int n_splits) {
    constexpr int PER = D / 32;
    // Launched as a programmatic dependent of the decode grid: wait here
    // until that grid has finished and its partials are visible.
    grid_dependency_wait();
    const long long row = static_cast<long long>(blockIdx.x) * 4 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const float* pl = part_lse + row * n_splits;
    float M = -INFINITY;
    for (int s = lane; s < n_splits; s += 32) M = fmaxf(M, pl[s]);
#pragma unroll
    for (int x = 16; x > 0; x >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, x));
    float L = 0.f;
    float acc[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) acc[i] = 0.f;
    const float* po = part_o + row * n_splits * D + lane * PER;
#pragma unroll 8
    for (int s = 0; s < n_splits; ++s) {
        const float ls = pl[s];
        const float w = ls == -INFINITY ? 0.f : ex2_approx(ls - M);
        L += w;
        if constexpr (PER == 4) {
            const float4 x = *reinterpret_cast<const float4*>(po + static_cast<long long>(s) * D);
            acc[0] += w * x.x;
            acc[1] += w * x.y;
            acc[2] += w * x.z;
            acc[3] += w * x.w;
        } else {
            const float2 x = *reinterpret_cast<const float2*>(po + static_cast<long long>(s) * D);
            acc[0] += w * x.x;
            acc[1] += w * x.y;
        }
    }
    const float inv = 1.f / L;
    __nv_bfloat16* orow = o + row * D + lane * PER;
    if constexpr (PER == 4) {
        uint2 packed;
        packed.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
        packed.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
        *reinterpret_cast<uint2*>(orow) = packed;
    } else {
        *reinterpret_cast<uint32_t*>(orow) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
    }
    if (lane == 0) lse[row] = (M + __log2f(L)) * 0.6931471805599453f;
}

}  // namespace fa
