// Block index maintenance: mean-pooling of key blocks (hisa_pool_blocks) and
// the per-token append (hisa_append).
//
// HISA (gptget.net summary, "Methodology"; Chinese summary, method details):
// the prefix is cut into contiguous blocks of B tokens and each block's keys
// are mean-pooled into one representative.  The blog ("Hierarchical Indexing
// Makes Sparse Attention Actually Fast", "HISA's Approach") keeps the summary
// current as tokens are appended; here only the trailing block changes.
//
// Both kernels run the same block_mean routine with the same thread mapping,
// so an appended block equals a from-scratch re-pool bit for bit.
#include "hisa_kernels.cuh"

namespace hisa {

namespace {

constexpr int kPoolThreads = 256;

// Geometry of one 16-byte vector of keys.
template <int D, bool E4M3>
struct PoolShape {
    static constexpr int kVec = E4M3 ? 16 : 8;             // elements per 16 B
    static constexpr int kLanes = D / kVec;                 // 16-B vectors per row
    static constexpr int kGroups = kPoolThreads / kLanes;   // rows read in parallel
};

__device__ __forceinline__ void dequant16(const uint4 raw, float scale, float (&v)[16]) {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const __nv_fp8x2_storage_t lo = static_cast<__nv_fp8x2_storage_t>(w[q] & 0xFFFFu);
        const __nv_fp8x2_storage_t hi = static_cast<__nv_fp8x2_storage_t>(w[q] >> 16);
        const float2 a = __half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2(lo, __NV_E4M3)));
        const float2 b = __half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2(hi, __NV_E4M3)));
        v[4 * q + 0] = a.x * scale;
        v[4 * q + 1] = a.y * scale;
        v[4 * q + 2] = b.x * scale;
        v[4 * q + 3] = b.y * scale;
    }
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
// pooled row and its hi/lo split.  fp32 sums: each thread adds its rows in
// order, then the per-group partial sums are added in group order.  The
// maximum is exact whatever the order.
template <int D, bool E4M3, bool MAX>
__device__ void block_mean(const KvView& kv, int b, int j, int s0, int cnt, float* partial) {
    using S = PoolShape<D, E4M3>;
    constexpr int V = S::kVec;
    const int tid = threadIdx.x;
    const int lane = tid % S::kLanes;
    const int grp = tid / S::kLanes;
    float acc[V];
#pragma unroll
    for (int e = 0; e < V; ++e) acc[e] = MAX ? -INFINITY : 0.f;

    const size_t row0 = static_cast<size_t>(b) * kv.cap + s0;
    if constexpr (E4M3) {
        const uint8_t* base = static_cast<const uint8_t*>(kv.keys);
        for (int r = grp; r < cnt; r += S::kGroups) {
            const uint4 raw = *reinterpret_cast<const uint4*>(base + (row0 + r) * D + lane * V);
            const float sc = kv.key_scale[row0 + r];
            float v[16];
            dequant16(raw, sc, v);
#pragma unroll
            for (int e = 0; e < V; ++e) acc[e] = MAX ? fmaxf(acc[e], v[e]) : acc[e] + v[e];
        }
    } else {
        const uint16_t* base = static_cast<const uint16_t*>(kv.keys);
        for (int r = grp; r < cnt; r += S::kGroups) {
            const uint4 raw = *reinterpret_cast<const uint4*>(base + (row0 + r) * D + lane * V);
            float v[8];
            bf16x8(raw, v);
#pragma unroll
            for (int e = 0; e < V; ++e) acc[e] = MAX ? fmaxf(acc[e], v[e]) : acc[e] + v[e];
        }
    }
#pragma unroll
    for (int e = 0; e < V; ++e) partial[grp * D + lane * V + e] = acc[e];
    __syncthreads();
    if (tid < D) {
        float sum = MAX ? -INFINITY : 0.f;
        for (int g = 0; g < S::kGroups; ++g)
            sum = MAX ? fmaxf(sum, partial[g * D + tid]) : sum + partial[g * D + tid];
        const float mean = MAX ? sum : sum / static_cast<float>(cnt);
        const size_t prow = static_cast<size_t>(b) * kv.nblk + j;
        kv.pooled[prow * D + tid] = mean;
        const __nv_bfloat16 hi = __float2bfloat16_rn(mean);
        const __nv_bfloat16 lo = __float2bfloat16_rn(mean - __bfloat162float(hi));
        __nv_bfloat16* hl = reinterpret_cast<__nv_bfloat16*>(kv.pooled_hl) + prow * 2 * D;
        hl[tid] = hi;
        hl[D + tid] = lo;
    }
}

template <int D, bool E4M3, bool MAX>
__global__ void __launch_bounds__(kPoolThreads) pool_kernel(KvView kv) {
    __shared__ __align__(16) float partial[PoolShape<D, E4M3>::kGroups * D];
    const int j = blockIdx.x;
    const int b = blockIdx.y;
    const int n = kv.len[b];
    if (n < 0 || n > kv.cap) {
        if (threadIdx.x == 0 && j == 0) set_status(kv.status, HISA_DEV_BAD_LEN);
        return;
    }
    const int s0 = j * kv.B;
    if (s0 >= n) return;
    const int cnt = min(kv.B, n - s0);
    block_mean<D, E4M3, MAX>(kv, b, j, s0, cnt, partial);
}

template <int D, bool E4M3, bool MAX>
__global__ void __launch_bounds__(kPoolThreads) append_kernel(KvView kv, const void* tok,
                                                              const float* tok_scale) {
    __shared__ __align__(16) float partial[PoolShape<D, E4M3>::kGroups * D];
    const int b = blockIdx.x;
    const int pos = kv.len[b];
    if (pos < 0 || pos >= kv.cap) {
        if (threadIdx.x == 0)
            set_status(kv.status, pos == kv.cap ? HISA_DEV_CAPACITY : HISA_DEV_BAD_LEN);
        return;
    }
    // 1. write the new key row (and its scale)
    constexpr int kRowBytes = D * (E4M3 ? 1 : 2);
    const size_t row = static_cast<size_t>(b) * kv.cap + pos;
    if (threadIdx.x < kRowBytes / 16) {
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(tok) +
                                                          static_cast<size_t>(b) * kRowBytes);
        uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(kv.keys) + row * kRowBytes);
        dst[threadIdx.x] = src[threadIdx.x];
    }
    if (E4M3 && threadIdx.x == 0) kv.key_scale[row] = tok_scale[b];
    __syncthreads();   // the row is visible to the whole block from here on
    // 2. recompute the trailing block over its valid keys
    const int j = pos / kv.B;
    const int s0 = j * kv.B;
    block_mean<D, E4M3, MAX>(kv, b, j, s0, pos - s0 + 1, partial);
    __syncthreads();
    // 3. publish the new length
    if (threadIdx.x == 0) kv.len[b] = pos + 1;
}

// Re-pool the trailing block of each sequence (the block holding key
// len - 1), e.g. a coarser index over keys another index's append just grew.
template <int D, bool E4M3, bool MAX>
__global__ void __launch_bounds__(kPoolThreads) tail_kernel(KvView kv) {
    __shared__ __align__(16) float partial[PoolShape<D, E4M3>::kGroups * D];
    const int b = blockIdx.x;
    const int n = kv.len[b];
    if (n < 0 || n > kv.cap) {
        if (threadIdx.x == 0) set_status(kv.status, HISA_DEV_BAD_LEN);
        return;
    }
    if (n == 0) return;
    const int j = (n - 1) / kv.B;
    const int s0 = j * kv.B;
    block_mean<D, E4M3, MAX>(kv, b, j, s0, n - s0, partial);
}

template <int D, bool E4M3>
cudaError_t launch_tail_t(const KvView& kv, cudaStream_t s) {
    if (kv.pool_max) tail_kernel<D, E4M3, true><<<kv.batch, kPoolThreads, 0, s>>>(kv);
    else tail_kernel<D, E4M3, false><<<kv.batch, kPoolThreads, 0, s>>>(kv);
    return cudaGetLastError();
}

template <int D, bool E4M3>
cudaError_t launch_pool_t(const KvView& kv, cudaStream_t s) {
    dim3 grid(kv.nblk, kv.batch);
    if (kv.pool_max) pool_kernel<D, E4M3, true><<<grid, kPoolThreads, 0, s>>>(kv);
    else pool_kernel<D, E4M3, false><<<grid, kPoolThreads, 0, s>>>(kv);
    return cudaGetLastError();
}

template <int D, bool E4M3>
cudaError_t launch_append_t(const KvView& kv, const void* tok, const float* tok_scale,
                            cudaStream_t s) {
    if (kv.pool_max) append_kernel<D, E4M3, true><<<kv.batch, kPoolThreads, 0, s>>>(kv, tok, tok_scale);
    else append_kernel<D, E4M3, false><<<kv.batch, kPoolThreads, 0, s>>>(kv, tok, tok_scale);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pool_tail(const KvView& kv, cudaStream_t s) {
    if (kv.d == 128) return kv.e4m3 ? launch_tail_t<128, true>(kv, s) : launch_tail_t<128, false>(kv, s);
    return kv.e4m3 ? launch_tail_t<64, true>(kv, s) : launch_tail_t<64, false>(kv, s);
}

cudaError_t launch_pool(const KvView& kv, cudaStream_t s) {
    if (kv.d == 128) return kv.e4m3 ? launch_pool_t<128, true>(kv, s) : launch_pool_t<128, false>(kv, s);
    return kv.e4m3 ? launch_pool_t<64, true>(kv, s) : launch_pool_t<64, false>(kv, s);
}

cudaError_t launch_append(const KvView& kv, const void* tok, const float* tok_scale,
                          cudaStream_t s) {
    if (kv.d == 128)
        return kv.e4m3 ? launch_append_t<128, true>(kv, tok, tok_scale, s)
                       : launch_append_t<128, false>(kv, tok, tok_scale, s);
    return kv.e4m3 ? launch_append_t<64, true>(kv, tok, tok_scale, s)
                   : launch_append_t<64, false>(kv, tok, tok_scale, s);
}

}  // namespace hisa
