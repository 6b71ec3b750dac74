// Block representatives (HISA: mean pooling of each block of B keys; gptget.net
// summary, "Methodology"), shared by the pool, append and trailing-block
// kernels, so that every path computes a block's representative with the
// same arithmetic and gets the same bits.
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

struct CtaSync {
    __device__ __forceinline__ void operator()() const { __syncthreads(); }
};

// Row rr of the block starting at cache row row0: this lane's 16-byte slice
// and (e4m3) the row's scale.
template <int D, bool E4M3>
__device__ __forceinline__ void mean_load(const KvView& kv, size_t row0, int rr, int lane, uint4& raw, float& sc) {
    constexpr int V = PoolShape<D, E4M3>::kVec;
    if constexpr (E4M3) {
        raw = *reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(kv.keys) + (row0 + rr) * D + lane * V);
        sc = kv.key_scale[row0 + rr];
    } else {
        raw = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(kv.keys) + (row0 + rr) * D + lane * V);
    }
}

// acc (+)= one row's slice (e4m3: acc = fma(x, scale, acc); max: of x * scale).
template <int D, bool E4M3, bool MAX>
__device__ __forceinline__ void mean_add(const uint4& raw, float sc, float (&acc)[PoolShape<D, E4M3>::kVec]) {
    constexpr int V = PoolShape<D, E4M3>::kVec;
    float x[V];
    if constexpr (E4M3) {
        e4m3x16(raw, *reinterpret_cast<float(*)[16]>(x));
        if constexpr (MAX) {
#pragma unroll
            for (int e = 0; e < V; ++e) acc[e] = fmaxf(acc[e], x[e] * sc);
        } else {
#pragma unroll
            for (int e = 0; e < V; e += 2) fma2_scaled(acc[e], acc[e + 1], x[e], x[e + 1], sc);
        }
    } else {
        bf16x8(raw, *reinterpret_cast<float(*)[8]>(x));
#pragma unroll
        for (int e = 0; e < V; ++e) acc[e] = MAX ? fmaxf(acc[e], x[e]) : acc[e] + x[e];
    }
}

// The group partial sums of each element added in group order, divided by
// cnt (or their maximum), into pooled row (b, j) and its hi/lo split.
template <int D, bool E4M3, bool MAX, int NT>
__device__ __forceinline__ void mean_finish(const KvView& kv, int b, int j, int cnt, const float* partial, int tid) {
    using S = PoolShape<D, E4M3>;
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

// Mean (or, MAX, elementwise maximum) of keys [s0, s0 + cnt) of sequence b ->
// pooled row and its hi/lo split.  The arithmetic is that of kPoolThreads
// "virtual" threads: virtual thread v (group v / kLanes, lane v % kLanes)
// adds, in fp32 and in row order, the rows grp, grp + kGroups, ... of its
// 16-byte column slice (an e4m3 row as acc = fma(x, scale, acc)); then
// mean_finish adds the group partial sums of each element in group order and
// divides by cnt.  NT real threads (NT divides kPoolThreads) play
// the virtual threads v = tid, tid + NT, ..., so every NT gives the same
// bits; `sync` is the barrier among the NT threads.  The loads of a chunk of
// rows for all of a thread's virtual threads are issued before their
// arithmetic, so that many are in flight at once.  The maximum is exact
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
                if (rr < cnt) mean_load<D, E4M3>(kv, row0, rr, lane[u], raw[u][i], sc[u][i]);
            }
#pragma unroll
        for (int u = 0; u < NV; ++u)
#pragma unroll
            for (int i = 0; i < kUnroll; ++i) {
                if (grp[u] + (i0 + i) * S::kGroups >= cnt) break;
                mean_add<D, E4M3, MAX>(raw[u][i], sc[u][i], acc[u]);
            }
    }
#pragma unroll
    for (int u = 0; u < NV; ++u)
#pragma unroll
        for (int e = 0; e < V; ++e) partial[grp[u] * D + lane[u] * V + e] = acc[u][e];
    sync();
    mean_finish<D, E4M3, MAX, NT>(kv, b, j, cnt, partial, tid);
}

// Rows a thread of block_mean (NT = kPoolThreads) reads in its single chunk.
template <int D, bool E4M3>
__host__ __device__ constexpr int pool_chunk_rows() {
    return PoolShape<D, E4M3>::kGroups * (!E4M3 ? 8 : 4);
}

// Blocks j and j + 1 of sequence b (cnt0 > 0 and cnt1 >= 0 keys, each at most
// pool_chunk_rows: one chunk), with block_mean's arithmetic for each; the
// rows of both are loaded before either is added, twice the bytes in flight,
// and the two blocks' group sums (partial holds 2 x kGroups x D floats) are
// reduced side by side, threads 0 .. NT/2 - 1 for the first block.
template <int D, bool E4M3, bool MAX>
__device__ void block_mean_pair(const KvView& kv, int b, int j, int s0, int cnt0, int cnt1, float* partial,
                                int tid) {
    using S = PoolShape<D, E4M3>;
    constexpr int V = S::kVec;
    constexpr int kUnroll = !E4M3 ? 8 : 4;
    static_assert(kPoolThreads / 2 >= D, "one reducing thread per element of each block");
    const int lane = tid % S::kLanes, grp = tid / S::kLanes;
    const int cnt[2] = {cnt0, cnt1};
    uint4 raw[2][kUnroll];
    float sc[2][kUnroll];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        const size_t row0 = static_cast<size_t>(b) * kv.cap + s0 + q * kv.B;
#pragma unroll
        for (int i = 0; i < kUnroll; ++i) {
            const int rr = grp + i * S::kGroups;
            raw[q][i] = make_uint4(0u, 0u, 0u, 0u);
            sc[q][i] = 1.f;
            if (rr < cnt[q]) mean_load<D, E4M3>(kv, row0, rr, lane, raw[q][i], sc[q][i]);
        }
    }
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        float acc[V];
#pragma unroll
        for (int e = 0; e < V; ++e) acc[e] = MAX ? -INFINITY : 0.f;
#pragma unroll
        for (int i = 0; i < kUnroll; ++i) {
            if (grp + i * S::kGroups >= cnt[q]) break;
            mean_add<D, E4M3, MAX>(raw[q][i], sc[q][i], acc);
        }
#pragma unroll
        for (int e = 0; e < V; ++e) partial[(q * S::kGroups + grp) * D + lane * V + e] = acc[e];
    }
    __syncthreads();
    const int q = tid / (kPoolThreads / 2);
    if (cnt[q] > 0)
        mean_finish<D, E4M3, MAX, kPoolThreads / 2>(kv, b, j + q, cnt[q], partial + q * S::kGroups * D,
                                                    tid - q * (kPoolThreads / 2));
}



// Shared-memory floats block_mean needs for its group partial sums.
__host__ __device__ constexpr int pool_partial_floats(int d, bool e4m3) {
    return kPoolThreads / (d / (e4m3 ? 16 : 8)) * d;
}

}  // namespace hisa
