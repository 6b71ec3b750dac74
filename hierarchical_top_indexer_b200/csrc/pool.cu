// Block index maintenance: mean-pooling of key blocks (hisa_pool_blocks) and
// the per-token append (hisa_append).
//
// HISA (gptget.net summary, "Methodology"; Chinese summary, method details):
// the prefix is cut into contiguous blocks of B tokens and each block's keys
// are mean-pooled into one representative.  The blog ("Hierarchical Indexing
// Makes Sparse Attention Actually Fast", "HISA's Approach") keeps the summary
// current as tokens are appended; here only the trailing block changes.
//
// Every kernel here (the decode step's append included) runs block_mean's
// arithmetic, so an appended block equals a from-scratch re-pool bit for
// bit.
#include "hisa_pool.cuh"

namespace hisa {

namespace {

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
    block_mean<D, E4M3, MAX, kPoolThreads>(kv, b, j, s0, cnt, partial, threadIdx.x, CtaSync{});
}

// e4m3 keys, blocks of one chunk: a CTA pools blocks 2x and 2x + 1, the
// rows of both loaded before either is added (an e4m3 block is half the
// bytes of a bf16 one, and four CTAs per SM would leave too few bytes in
// flight).  Each block's arithmetic is block_mean's.
template <int D, bool MAX>
__global__ void __launch_bounds__(kPoolThreads) pool_pair_kernel(KvView kv) {
    __shared__ __align__(16) float partial[2 * PoolShape<D, true>::kGroups * D];
    const int j = 2 * blockIdx.x;
    const int b = blockIdx.y;
    const int n = kv.len[b];
    if (n < 0 || n > kv.cap) {
        if (threadIdx.x == 0 && j == 0) set_status(kv.status, HISA_DEV_BAD_LEN);
        return;
    }
    const int s0 = j * kv.B;
    if (s0 >= n) return;
    const int cnt0 = min(kv.B, n - s0);
    const int cnt1 = j + 1 < kv.nblk && s0 + kv.B < n ? min(kv.B, n - s0 - kv.B) : 0;
    block_mean_pair<D, true, MAX>(kv, b, j, s0, cnt0, cnt1, partial, threadIdx.x);
}

// STEP: the decode step's append (launched with programmatic dependent
// launch): the next kernel, which scores this step's blocks, may start at once
// (it reads the old length and takes the new key's position from it); the
// length is advanced by that kernel after it has waited for this one.
template <int D, bool E4M3, bool MAX, bool STEP>
__global__ void __launch_bounds__(kPoolThreads) append_kernel(KvView kv, const void* tok,
                                                              const float* tok_scale) {
    __shared__ __align__(16) float partial[PoolShape<D, E4M3>::kGroups * D];
    if (STEP) {
        grid_dependency_wait();
        grid_launch_dependents();
    }
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
    block_mean<D, E4M3, MAX, kPoolThreads>(kv, b, j, s0, pos - s0 + 1, partial, threadIdx.x, CtaSync{});
    __syncthreads();
    // 3. publish the new length (the decode step's scoring kernel does it)
    if (!STEP && threadIdx.x == 0) kv.len[b] = pos + 1;
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
    block_mean<D, E4M3, MAX, kPoolThreads>(kv, b, j, s0, n - s0, partial, threadIdx.x, CtaSync{});
}

template <int D, bool E4M3>
cudaError_t launch_tail_t(const KvView& kv, cudaStream_t s) {
    if (kv.pool_max) tail_kernel<D, E4M3, true><<<kv.batch, kPoolThreads, 0, s>>>(kv);
    else tail_kernel<D, E4M3, false><<<kv.batch, kPoolThreads, 0, s>>>(kv);
    return cudaGetLastError();
}

template <int D, bool E4M3>
cudaError_t launch_pool_t(const KvView& kv, cudaStream_t s) {
    if (E4M3 && kv.B <= pool_chunk_rows<D, true>()) {
        dim3 grid((kv.nblk + 1) / 2, kv.batch);
        if (kv.pool_max) pool_pair_kernel<D, true><<<grid, kPoolThreads, 0, s>>>(kv);
        else pool_pair_kernel<D, false><<<grid, kPoolThreads, 0, s>>>(kv);
        return cudaGetLastError();
    }
    dim3 grid(kv.nblk, kv.batch);
    if (kv.pool_max) pool_kernel<D, E4M3, true><<<grid, kPoolThreads, 0, s>>>(kv);
    else pool_kernel<D, E4M3, false><<<grid, kPoolThreads, 0, s>>>(kv);
    return cudaGetLastError();
}

template <int D, bool E4M3, bool STEP>
cudaError_t launch_append_s(const KvView& kv, const void* tok, const float* tok_scale, cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(kv.batch));
    cfg.blockDim = dim3(kPoolThreads);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = STEP ? 1 : 0;
    const cudaError_t e = kv.pool_max
        ? cudaLaunchKernelEx(&cfg, append_kernel<D, E4M3, true, STEP>, kv, tok, tok_scale)
        : cudaLaunchKernelEx(&cfg, append_kernel<D, E4M3, false, STEP>, kv, tok, tok_scale);
    return e != cudaSuccess ? e : cudaGetLastError();
}

template <int D, bool E4M3>
cudaError_t launch_append_t(const KvView& kv, const void* tok, const float* tok_scale, bool step,
                            cudaStream_t s) {
    return step ? launch_append_s<D, E4M3, true>(kv, tok, tok_scale, s)
                : launch_append_s<D, E4M3, false>(kv, tok, tok_scale, s);
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
                          cudaStream_t s, bool step) {
    if (kv.d == 128)
        return kv.e4m3 ? launch_append_t<128, true>(kv, tok, tok_scale, step, s)
                       : launch_append_t<128, false>(kv, tok, tok_scale, step, s);
    return kv.e4m3 ? launch_append_t<64, true>(kv, tok, tok_scale, step, s)
                   : launch_append_t<64, false>(kv, tok, tok_scale, step, s);
}

}  // namespace hisa
