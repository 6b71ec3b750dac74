// Block representatives (HISA: mean pooling of each block of B keys; gptget.net
// summary, "Methodology"), shared by the pool / append kernels and by the
// decode step fused into block scoring, so that every path computes a block's
// representative with the same arithmetic and gets the same bits.
#pragma once

#include "hisa_kernels.cuh"

namespace hisa {

constexpr int kPoolThreads = 256;   // virtual threads of block_mean

// Geometry of one 16-byte vector of keys.
template <int D, bool E4M3>
struct PoolShape {
    static constexpr int kVec = E4M3 ? 16 : 8;             // elements per 16 B
    static constexpr int kLanes = D / kVec;                 // 16-B vectors per row
    static constexpr int kGroups = kPoolThreads / kLanes;   // rows read in parallel
};

// 16 e4m3 keys -> fp32 (exact), before the key's scale is applied.
__device__ __forceinline__ void e4m3x16(const uint4 raw, float (&v)[16]) {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const __nv_fp8x2_storage_t lo = static_cast<__nv_fp8x2_storage_t>(w[q] & 0xFFFFu);
        const __nv_fp8x2_storage_t hi = static_cast<__nv_fp8x2_storage_t>(w[q] >> 16);
        const float2 a = __half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2(lo, __NV_E4M3)));
        const float2 b = __half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2(hi, __NV_E4M3)));
        v[4 * q + 0] = a.x;
        v[4 * q + 1] = a.y;
        v[4 * q + 2] = b.x;
        v[4 * q + 3] = b.y;
    }
}

// a0 = fma(x0, s, a0) and a1 = fma(x1, s, a1) (one packed instruction).
__device__ __forceinline__ void fma2_scaled(float& a0, float& a1, float x0, float x1, float s) {
    fma2(a0, a1, x0, x1, s, s);
}

__device__ __forceinline__ void bf16x8(const uint4 raw, float (&v)[8]) {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        v[2 * q + 0] = __uint_as_float(w[q] << 16);
        v[2 * q + 1] = __uint_as_float(w[q] & 0xFFFF0000u);
    }
}

// Mean (or, MAX, elementwise maximum) of keys [s0, s0 + cnt) of sequence b ->
// pooled row and its hi/lo split.  The arithmetic is that of kPoolThreads
// "virtual" threads: virtual thread v (group v / kLanes, lane v % kLanes)
// adds, in fp32 and in row order, the rows grp, grp + kGroups, ... of its
// 16-byte column slice (an e4m3 row as acc = fma(x, scale, acc)); then the group partial sums of each element are added
// in group order and divided by cnt.  NT real threads (NT divides
// kPoolThreads) play the virtual threads v = tid, tid + NT, ..., so every NT
// gives the same bits; `sync` is the barrier among the NT threads.  The loads
// of a chunk of rows for all of a thread's virtual threads are issued before
// their arithmetic, so that many are in flight at once.  The maximum is exact
// whatever the order.
template <int D, bool E4M3, bool MAX, int NT, class Sync>
__device__ void block_mean(const KvView& kv, int b, int j, int s0, int cnt, float* partial, int tid,
                           Sync sync) {
    using S = PoolShape<D, E4M3>;
    constexpr int V = S::kVec;
    constexpr int NV = kPoolThreads / NT;          // virtual threads per thread
    // rows per virtual thread per chunk (e4m3 rows dequantise into twice the
    // registers: a shorter chunk keeps the pool kernel's occupancy)
    constexpr int kUnroll = NV == 1 && !E4M3 ? 8 : 4;
    static_assert(kPoolThreads % NT == 0, "virtual threads split evenly");
    const size_t row0 = static_cast<size_t>(b) * kv.cap + s0;
    int lane[NV], grp[NV];
    float acc[NV][V];
#pragma unroll
    for (int u = 0; u < NV; ++u) {
        const int v = tid + u * NT;
        lane[u] = v % S::kLanes;
        grp[u] = v / S::kLanes;
#pragma unroll
        for (int e = 0; e < V; ++e) acc[u][e] = MAX ? -INFINITY : 0.f;
    }
    // virtual thread u adds rows grp[u] + i * kGroups, i = 0, 1, ... in order;
    // a chunk issues kUnroll of them for every u before any arithmetic
    for (int i0 = 0; grp[0] + i0 * S::kGroups < cnt; i0 += kUnroll) {
        uint4 raw[NV][kUnroll];
        float sc[NV][kUnroll];
#pragma unroll
        for (int u = 0; u < NV; ++u)
#pragma unroll
            for (int i = 0; i < kUnroll; ++i) {
                const int rr = grp[u] + (i0 + i) * S::kGroups;
                raw[u][i] = make_uint4(0u, 0u, 0u, 0u);
                sc[u][i] = 1.f;
                if (rr < cnt) {
                    if constexpr (E4M3) {
                        raw[u][i] = *reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(kv.keys) +
                                                                    (row0 + rr) * D + lane[u] * V);
                        sc[u][i] = kv.key_scale[row0 + rr];
                    } else {
                        raw[u][i] = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(kv.keys) +
                                                                    (row0 + rr) * D + lane[u] * V);
                    }
                }
            }
#pragma unroll
        for (int u = 0; u < NV; ++u)
#pragma unroll
            for (int i = 0; i < kUnroll; ++i) {
                if (grp[u] + (i0 + i) * S::kGroups >= cnt) break;
                float x[V];
                if constexpr (E4M3) {
                    // sum: acc + x * scale as one fma per element; max: of x * scale
                    e4m3x16(raw[u][i], *reinterpret_cast<float(*)[16]>(x));
                    if constexpr (MAX) {
#pragma unroll
                        for (int e = 0; e < V; ++e) acc[u][e] = fmaxf(acc[u][e], x[e] * sc[u][i]);
                    } else {
#pragma unroll
                        for (int e = 0; e < V; e += 2)
                            fma2_scaled(acc[u][e], acc[u][e + 1], x[e], x[e + 1], sc[u][i]);
                    }
                } else {
                    bf16x8(raw[u][i], *reinterpret_cast<float(*)[8]>(x));
#pragma unroll
                    for (int e = 0; e < V; ++e) acc[u][e] = MAX ? fmaxf(acc[u][e], x[e]) : acc[u][e] + x[e];
                }
            }
    }
#pragma unroll
    for (int u = 0; u < NV; ++u)
#pragma unroll
        for (int e = 0; e < V; ++e) partial[grp[u] * D + lane[u] * V + e] = acc[u][e];
    sync();
    for (int x = tid; x < D; x += NT) {
        float sum = MAX ? -INFINITY : 0.f;
        for (int g = 0; g < S::kGroups; ++g)
            sum = MAX ? fmaxf(sum, partial[g * D + x]) : sum + partial[g * D + x];
        const float mean = MAX ? sum : sum / static_cast<float>(cnt);
        const size_t prow = static_cast<size_t>(b) * kv.nblk + j;
        kv.pooled[prow * D + x] = mean;
        const __nv_bfloat16 hi = __float2bfloat16_rn(mean);
        const __nv_bfloat16 lo = __float2bfloat16_rn(mean - __bfloat162float(hi));
        __nv_bfloat16* hl = reinterpret_cast<__nv_bfloat16*>(kv.pooled_hl) + prow * 2 * D;
        hl[x] = hi;
        hl[D + x] = lo;
    }
}

struct CtaSync {
    __device__ __forceinline__ void operator()() const { __syncthreads(); }
};

// Shared-memory floats block_mean needs for its group partial sums.
__host__ __device__ constexpr int pool_partial_floats(int d, bool e4m3) {
    return kPoolThreads / (d / (e4m3 ? 16 : 8)) * d;
}

}  // namespace hisa
