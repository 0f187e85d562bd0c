// fa_merge_kernels.cuh -- combining attention computed over disjoint key
// sets, for sequence sharding across devices (Ring Attention).
//
// Ring Attention with Blockwise Transformers (abstract): the sequence is
// spread over a ring of devices; each device keeps its query block while the
// key/value blocks travel around the ring, and each block's attention is
// folded into the device's running result.  The folding is the same
// log-sum-exp rescaling that the online softmax applies block by block
// (iplexlaw FlashAttention-2 blog, "Tiling preserves the attention
// calculation"): for two partial results over disjoint key sets,
//     M = max(lse_a, lse_b),  w_a = exp(lse_a - M),  w_b = exp(lse_b - M),
//     O = (w_a O_a + w_b O_b) / (w_a + w_b),  LSE = M + log(w_a + w_b),
// which is exactly attention over the union of the two key sets.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "sm100_ptx.cuh"

namespace fa {

// One thread per 8 columns of a row.  init: the accumulator takes the
// partial as it is.  o_out (may be null): bf16 copy of the merged row.
template <int D>
__global__ void __launch_bounds__(256) fa_lse_merge_kernel(
    float* __restrict__ o_acc, float* __restrict__ lse_acc,
    const __nv_bfloat16* __restrict__ o_part, const float* __restrict__ lse_part,
    __nv_bfloat16* __restrict__ o_out, long long rows, int init) {
    constexpr int G = D / 8;
    const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    const long long row = gid / G;
    if (row >= rows) return;
    const int col = static_cast<int>(gid % G) * 8;
    const long long off = row * D + col;
    const uint4 pb = *reinterpret_cast<const uint4*>(o_part + off);
    const uint32_t pw[4] = {pb.x, pb.y, pb.z, pb.w};
    float part[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        part[2 * i] = __uint_as_float(pw[i] << 16);
        part[2 * i + 1] = __uint_as_float(pw[i] & 0xffff0000u);
    }
    const float lb = lse_part[row];
    float out[8];
    float lse_new;
    if (init) {
#pragma unroll
        for (int i = 0; i < 8; ++i) out[i] = part[i];
        lse_new = lb;
    } else {
        const float la = lse_acc[row];
        const float4* pa = reinterpret_cast<const float4*>(o_acc + off);
        const float4 a0 = pa[0], a1 = pa[1];
        const float acc[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        const float M = fmaxf(la, lb);
        if (M == -INFINITY) {  // neither side saw a key: keep the accumulator
#pragma unroll
            for (int i = 0; i < 8; ++i) out[i] = acc[i];
            lse_new = la;
        } else {
            const float wa = expf(la - M), wb = expf(lb - M);
            const float inv = 1.0f / (wa + wb);
#pragma unroll
            for (int i = 0; i < 8; ++i) out[i] = (wa * acc[i] + wb * part[i]) * inv;
            lse_new = M + logf(wa + wb);
        }
    }
    float4* pa = reinterpret_cast<float4*>(o_acc + off);
    pa[0] = make_float4(out[0], out[1], out[2], out[3]);
    pa[1] = make_float4(out[4], out[5], out[6], out[7]);
    if (col == 0) lse_acc[row] = lse_new;
    if (o_out) {
        uint4 ob;
        ob.x = pack_bf16x2(out[0], out[1]);
        ob.y = pack_bf16x2(out[2], out[3]);
        ob.z = pack_bf16x2(out[4], out[5]);
        ob.w = pack_bf16x2(out[6], out[7]);
        *reinterpret_cast<uint4*>(o_out + off) = ob;
    }
}

// dst = bf16(src), 8 elements per thread.
__global__ void __launch_bounds__(256) fa_f32_to_bf16_kernel(const float* __restrict__ src,
                                                             __nv_bfloat16* __restrict__ dst,
                                                             long long n8) {
    const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= n8) return;
    const float4* s = reinterpret_cast<const float4*>(src) + 2 * i;
    const float4 a = s[0], b = s[1];
    uint4 o;
    o.x = pack_bf16x2(a.x, a.y);
    o.y = pack_bf16x2(a.z, a.w);
    o.z = pack_bf16x2(b.x, b.y);
    o.w = pack_bf16x2(b.z, b.w);
    reinterpret_cast<uint4*>(dst)[i] = o;
}

}  // namespace fa
