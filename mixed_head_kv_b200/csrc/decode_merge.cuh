// decode_merge.cuh — the split-KV merge of a decode step (D4), shared by the
// CUDA-core and tensor-core decode kernels: the last CTA of a (sequence, KV
// head) combines the splits' normalised partial outputs by their log2-sum-exp2
// weights, o = sum_s 2^(lse_s - M) o_s / sum_s 2^(lse_s - M).
#pragma once

#include "duo_internal.cuh"
#include "sm100.cuh"

namespace duo {

// The split handshake, by every thread of a CTA that has stored its partial:
// the stores precede (a barrier, then thread 0's GPU-scope acq_rel fence) the
// increment of the (sequence, KV head) counter; the CTA whose increment
// completes the count acquires the other CTAs' partials (the same fence after
// the increment, then a barrier) and returns true: it merges.
__device__ __forceinline__ bool split_arrive(uint32_t* counter, uint32_t nsplit, volatile int* flag) {
    __syncthreads();
    if (threadIdx.x == 0) {
        asm volatile("fence.acq_rel.gpu;" ::: "memory");
        const bool last = atomicAdd(counter, 1u) == nsplit - 1;
        if (last) asm volatile("fence.acq_rel.gpu;" ::: "memory");
        *flag = last ? 1 : 0;
    }
    __syncthreads();
    return *flag != 0;
}

// Called by every thread of the merging CTA (kThreads of them) after a barrier;
// `smem` holds kThreads float4 + 2 * kThreads floats of scratch at least.
// The partials of this (b, KV head) are contiguous: [nsplit][G][D] floats and
// [nsplit][G] log-sum-exps. Thread (rep, unit) merges the splits rep, rep +
// kRep, ... of one float4 unit online (running max, weight sum, weighted sum),
// issuing the loads of up to kChunk splits (partials and log-sum-exps) at once,
// so the merge costs about one round trip to L2 rather than one per phase; the
// kRep partial merges of a unit are then combined through shared memory.
template <int G, int D, int kThreads>
__device__ __forceinline__ void merge_split_partials(const DecodeParams& p, int b, int g, int ri, uint8_t* smem) {
    const int tid = threadIdx.x;
    const int64_t item0 = (static_cast<int64_t>(b) * p.n_retr + ri) * p.nsplit;
    const int ns = p.nsplit;
    constexpr int kUnits = G * D / 4;  // float4 units of one split's partial
    constexpr int kRep = kUnits >= kThreads ? 1 : kThreads / kUnits;
    constexpr int kChunk = kRep >= 4 ? 16 : (kRep == 2 ? 8 : 4);  // splits per batch of loads (register budget)
    float4* sm_acc = reinterpret_cast<float4*>(smem);                 // [kRep][kUnits]
    float* sm_mm = reinterpret_cast<float*>(sm_acc + kRep * kUnits);  // [kRep][kUnits] max
    float* sm_ll = sm_mm + kRep * kUnits;                             // [kRep][kUnits] weight sum
    const float4* po = reinterpret_cast<const float4*>(p.part_o + item0 * G * D);
    const float* pl = p.part_lse + item0 * G;
    const bool in_rep = tid / kUnits < kRep;
    const int rep = in_rep ? tid / kUnits : 0;
    for (int u = tid % kUnits; in_rep && u < kUnits; u += kThreads) {
        const int h = (u * 4) / D;
        float M = -INFINITY, Ls = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int sp0 = rep; sp0 < ns; sp0 += kRep * kChunk) {
            float x[kChunk];
            float4 o[kChunk];
#pragma unroll
            for (int k = 0; k < kChunk; ++k) {
                const int sp = sp0 + k * kRep;
                x[k] = sp < ns ? __ldcg(pl + sp * G + h) : -INFINITY;
                o[k] = sp < ns ? __ldcg(po + static_cast<int64_t>(sp) * kUnits + u) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int k = 0; k < kChunk; ++k) {
                if (x[k] == -INFINITY) continue;  // a split without rows, or past the last split
                if (x[k] > M) {
                    const float f = fast_exp2(M - x[k]);  // 0 while M is -inf
                    Ls *= f;
                    acc.x *= f;
                    acc.y *= f;
                    acc.z *= f;
                    acc.w *= f;
                    M = x[k];
                }
                const float w = fast_exp2(x[k] - M);
                Ls += w;
                acc.x = fmaf(w, o[k].x, acc.x);
                acc.y = fmaf(w, o[k].y, acc.y);
                acc.z = fmaf(w, o[k].z, acc.z);
                acc.w = fmaf(w, o[k].w, acc.w);
            }
        }
        sm_acc[rep * kUnits + u] = acc;
        sm_mm[rep * kUnits + u] = M;
        sm_ll[rep * kUnits + u] = Ls;
    }
    __syncthreads();
    for (int u = tid; u < kUnits; u += kThreads) {
        float M = -INFINITY;
        for (int r = 0; r < kRep; ++r) M = fmaxf(M, sm_mm[r * kUnits + u]);
        float Ls = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int r = 0; r < kRep; ++r) {
            const float mr = sm_mm[r * kUnits + u];
            if (mr == -INFINITY) continue;
            const float f = fast_exp2(mr - M);
            const float4 x = sm_acc[r * kUnits + u];
            Ls = fmaf(f, sm_ll[r * kUnits + u], Ls);
            acc.x = fmaf(f, x.x, acc.x);
            acc.y = fmaf(f, x.y, acc.y);
            acc.z = fmaf(f, x.z, acc.z);
            acc.w = fmaf(f, x.w, acc.w);
        }
        const float inv = 1.f / Ls;  // Ls >= 1: the split holding the maximum weighs 1
        const int h = (u * 4) / D;
        const int d = (u * 4) % D;
        bf16* o = p.out + (static_cast<int64_t>(b) * p.Hq + g * G + h) * D + d;
        *reinterpret_cast<uint2*>(o) =
            make_uint2(pack_bf16x2(acc.x * inv, acc.y * inv), pack_bf16x2(acc.z * inv, acc.w * inv));
    }
}

}  // namespace duo
