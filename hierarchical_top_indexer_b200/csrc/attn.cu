// Sparse attention over the selected tokens: the operator HISA's indices feed.
//
// The selection exists so that attention reads only k tokens per query (HISA
// blog, "How Fine-Grained Sparse Attention Works Today": the second stage
// attends to the top-K tokens only; arXiv abstract: the indices go to the
// sparse attention operator).  This kernel is a synthetic consumer in the
// multi-query form such operators take: Ha query heads share one key head
// and one value head (d = 128 each), and for query row i
//     o[i, h] = sum_j softmax_j(scale * qa[i, h] . K[b, idx[i, j]]) V[b, idx[i, j]]
// over the entries j with 0 <= idx[i, j] < len[b] (the others are padding).
//
// Layout of one CTA (416 threads): warps 0-3 gather, warp 4 issues the
// tcgen05 MMAs, warps 5-12 run the softmax (two threads per head, one per
// half of the tile's 128 columns).  A CTA
// takes a contiguous range of (row, 128-token tile) slots; a run of tiles of
// one row is a segment, whose unnormalised output, running max and sum go to
// the workspace, and combine_kernel merges a row's segments.
//   gather:  per tile, the key and value rows (256 B each) of the tile's 128
//            tokens, by 16-byte cp.async into the 128-byte swizzled operand
//            layout, half a warp per row (zero rows for padding entries).
//   MMA:     S = Qa K^T (M = 128 heads, N = 128 tokens, K = 128) into one of
//            two TMEM buffers; then O += P V (K = 128 tokens, V read
//            MN-major) into a third.
//   softmax: per tile, the head's row of S: max, p = 2^(s - max) rounded to
//            bf16 into the P operand, running sum (of the unrounded p); when
//            the max grows, the head's row of O is rescaled in TMEM before
//            the next P V.
#include "hisa_kernels.cuh"

namespace hisa {

namespace {

constexpr int kAttnThreads = 416;
constexpr int kWarpMmaA = 4;    // warps 0-3 gather
constexpr int kWarpSoft0 = 5;   // warps 5-12 softmax
constexpr int kAttnStages = 2;
constexpr int kOperandBytes = 128 * 256;            // one 128 x 128 bf16 operand
constexpr int kAttnSmem = kOperandBytes * (2 + 2 * kAttnStages) + 1024 + 4096;

struct AttnLayout {
    static constexpr int q = 0;
    static constexpr int k0 = kOperandBytes;                       // K of stage s: k0 + s * 2 * op
    static constexpr int p = kOperandBytes * (1 + 2 * kAttnStages);
    static constexpr int bars = kOperandBytes * (2 + 2 * kAttnStages);
    static constexpr int red = bars + 256;         // [2][2][128] fp32 maxima of the halves
    static constexpr int lred = red + 2048;        // [2][128] fp32 sums of the halves
};

// Byte offset of 16-byte chunk c (0..15) of row r (0..127) of a 128 x 128
// bf16 operand in the 128-byte swizzled layout: two 64-column atoms of 16 KB,
// rows of 128 B, chunk index XOR (row mod 8).
__device__ __forceinline__ uint32_t sw128_off(int r, int c) {
    return static_cast<uint32_t>((c >> 3) * 16384 + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// 16-byte asynchronous copy global -> shared; src_bytes = 0 writes zeros.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
                 : "memory");
}

// 32 lanes x 32 bit, 16 consecutive columns per thread (TMEM store).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Descriptor of an MN-major operand in the 128-byte swizzled layout: atoms of
// 64 MN-elements x 8 K-rows (1 KB); the two 64-wide MN atoms are 16 KB apart
// (leading offset), consecutive 8-row K groups 1 KB apart (stride offset).
__device__ __forceinline__ uint64_t sw128_mnmajor_desc(uint32_t saddr) {
    return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(16384 >> 4) << 16) |
           (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
           (static_cast<uint64_t>(2) << 61);
}

// bf16 x bf16 -> fp32, M = N = 128, A K-major; B K-major or MN-major.
__host__ __device__ constexpr uint32_t idesc_attn(bool b_mn_major) {
    return idesc_bf16_f32(128) | (b_mn_major ? (1u << 16) : 0u);
}

// 2^x by the hardware approximation (about 2^-22 relative; 2^-inf = 0).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

struct Seg {
    int row, t0, n;   // row, first tile, tiles
};

// Segment of the range [g, g1) that starts at g (tiles of one row).
__device__ __forceinline__ Seg next_seg(long long g, long long g1, int T) {
    Seg s;
    s.row = static_cast<int>(g / T);
    s.t0 = static_cast<int>(g - static_cast<long long>(s.row) * T);
    const long long end = min(g1, static_cast<long long>(s.row + 1) * T);
    s.n = static_cast<int>(end - g);
    return s;
}

// Whether entry j of row i names a visible token of its sequence.
__device__ __forceinline__ bool attn_valid(const AttnParams& p, int row, int j, int len_b) {
    if (j >= p.k) return false;
    const int s = p.idx[static_cast<size_t>(row) * p.k + j];
    return s >= 0 && s < len_b;
}

__device__ __forceinline__ int seq_len(const AttnParams& p, int row, int* b_out) {
    const int b = p.q_seq[row];
    *b_out = b;
    if (b < 0 || b >= p.batch) return 0;
    const int n = p.len[b];
    return (n < 0 || n > p.cap) ? 0 : n;
}

// Lane 0 waits (bounded); the warp learns the outcome.
__device__ __forceinline__ bool warp_wait_a(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    bool ok = true;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort_flag);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    __syncwarp();
    return ok;
}

__device__ __forceinline__ void attn_abort(volatile int* abort_flag, uint32_t* status) {
    *abort_flag = 1;
    set_status(status, HISA_DEV_TIMEOUT);
}

__global__ void __launch_bounds__(kAttnThreads, 1) attn_kernel(const AttnParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + AttnLayout::bars);
    uint64_t* full = bars;                  // [stages] a tile's K and V landed (128 copy arrivals)
    uint64_t* empty = full + kAttnStages;   // [stages] the tile's P V is done (commit)
    uint64_t* sfull = empty + kAttnStages;  // [2] S buffer written (commit)
    uint64_t* sempty = sfull + 2;           // [2] S buffer read (8 softmax warps)
    uint64_t* qfull = sempty + 2;           // the segment's query heads landed (128 arrivals)
    uint64_t* qempty = qfull + 1;           // the segment's last S MMA is done (commit)
    uint64_t* pfull = qempty + 1;           // P written and O corrected (8 softmax warps)
    uint64_t* ofull = pfull + 1;            // a P V is done (commit)
    uint64_t* done = ofull + 1;             // every MMA issued is done (commit)
    uint64_t* xbar = done + 1;              // [2] both halves' maxima written (8 softmax warps)
    uint64_t* lbar = xbar + 2;              // both halves' sums written (8 softmax warps)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(lbar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = p.T;
    const long long total = static_cast<long long>(p.n_q) * T;
    const long long g0 = total * blockIdx.x / gridDim.x;
    const long long g1 = total * (blockIdx.x + 1) / gridDim.x;

    if (warp == kWarpMmaA) {
        if (lane == 0) {
            for (int s = 0; s < kAttnStages; ++s) {
                mbar_init(full + s, 128);
                mbar_init(empty + s, 1);
            }
            for (int b = 0; b < 2; ++b) {
                mbar_init(sfull + b, 1);
                mbar_init(sempty + b, 8);
                mbar_init(xbar + b, 8);
            }
            mbar_init(lbar, 8);
            mbar_init(qfull, 128);
            mbar_init(qempty, 1);
            mbar_init(pfull, 8);
            mbar_init(ofull, 1);
            mbar_init(done, 1);
            *abort_flag = 0;
            fence_barrier_init();
        }
        __syncwarp();
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    grid_dependency_wait();
    grid_launch_dependents();

    uint8_t* sQ = smem + AttnLayout::q;
    uint8_t* sP = smem + AttnLayout::p;

    if (warp < 4) {
        // ---------------------------------------------------------- gather
        // Warp w copies rows 32 w .. 32 w + 31 of each operand; one copy
        // instruction moves two whole 256-byte rows (lanes 0-15 the first,
        // 16-31 the second), so every request is a contiguous run.
        const int rbase = warp * 32;
        const int c = lane & 15;
        bool ok = true;
        int it = 0, qn = 0;
        for (long long g = g0; g < g1 && ok;) {
            const Seg sg = next_seg(g, g1, T);
            int b;
            const int len_b = seq_len(p, sg.row, &b);
            if (qn > 0 && !warp_wait_a(qempty, (qn - 1) & 1, abort_flag)) {
                ok = false;
                break;
            }
            {
                const uint32_t dst = smem_addr(sQ);
#pragma unroll 4
                for (int i = 0; i < 16; ++i) {
                    const int r = rbase + 2 * i + (lane >> 4);
                    const bool hv = r < p.Ha;
                    const uint16_t* src = p.q + (hv ? (static_cast<size_t>(sg.row) * p.Ha + r) * 128 + 8 * c : 0);
                    cp_async_16(dst + sw128_off(r, c), src, hv ? 16u : 0u);
                }
                cp_async_arrive_noinc(qfull);
            }
            ++qn;
            for (int j = 0; j < sg.n; ++j, ++it) {
                const int st = it % kAttnStages, use = it / kAttnStages;
                // this lane's token (row rbase + lane), read before the wait for a free stage
                const int slot = (sg.t0 + j) * 128 + rbase + lane;
                int tok = slot < p.k ? p.idx[static_cast<size_t>(sg.row) * p.k + slot] : -1;
                if (use > 0 && !warp_wait_a(empty + st, (use - 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                const bool v = tok >= 0 && tok < len_b;
                if (!v) tok = 0;
                const uint32_t dk = smem_addr(smem + AttnLayout::k0 + st * 2 * kOperandBytes);
                const uint32_t dv = dk + kOperandBytes;
#pragma unroll 4
                for (int i = 0; i < 16; ++i) {
                    // row rr's token and validity (not this lane's own)
                    const int rr = 2 * i + (lane >> 4);
                    const int t_i = __shfl_sync(0xffffffffu, tok, rr);
                    const bool v_i = __shfl_sync(0xffffffffu, v ? 1 : 0, rr) != 0;
                    const size_t off = (static_cast<size_t>(v_i ? b : 0) * p.cap + t_i) * 128 + 8 * c;
                    const uint32_t o = sw128_off(rbase + rr, c);
                    cp_async_16(dk + o, p.kc + off, v_i ? 16u : 0u);
                    cp_async_16(dv + o, p.vc + off, v_i ? 16u : 0u);
                }
                cp_async_arrive_noinc(full + st);
            }
            g += sg.n;
        }
        cp_async_wait_all();
    } else if (warp == kWarpMmaA) {
        // ------------------------------------------------------------- MMA
        if (lane == 0) {
            bool ok = true;
            uint32_t it = 0, sc = 0, pn = 0, qn = 0;
            const uint32_t id_s = idesc_attn(false), id_o = idesc_attn(true);
            const uint32_t aq = smem_addr(sQ), ap = smem_addr(sP);
            auto issue_s = [&](uint32_t tile) -> bool {
                const uint32_t st = tile % kAttnStages, use = tile / kAttnStages;
                if (!mbar_wait(full + st, use & 1, abort_flag)) return false;
                const uint32_t buf = sc & 1;
                if (sc >= 2 && !mbar_wait(sempty + buf, ((sc >> 1) - 1) & 1, abort_flag)) return false;
                // the tile arrived by cp.async (generic proxy); the MMAs read it through the async proxy
                fence_async_smem();
                tc_fence_after();
                const uint32_t bk = smem_addr(smem + AttnLayout::k0 + st * 2 * kOperandBytes);
#pragma unroll
                for (int s = 0; s < 8; ++s) {
                    const uint32_t o = (s >> 2) * 16384 + (s & 3) * 32;
                    umma_bf16(tmem_base + buf * 128, sw128_kmajor_desc(aq + o), sw128_kmajor_desc(bk + o), id_s,
                              s > 0);
                }
                umma_commit(sfull + buf);
                ++sc;
                return true;
            };
            for (long long g = g0; g < g1 && ok;) {
                const Seg sg = next_seg(g, g1, T);
                if (!mbar_wait(qfull, qn & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                ++qn;
                fence_async_smem();
                tc_fence_after();
                ok = issue_s(it);
                for (int j = 0; j < sg.n && ok; ++j) {
                    if (j + 1 < sg.n) ok = issue_s(it + j + 1);
                    else umma_commit(qempty);   // the segment's query heads are no longer read
                    if (!ok) break;
                    if (!mbar_wait(pfull, pn & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    ++pn;
                    tc_fence_after();
                    const uint32_t st = (it + j) % kAttnStages;
                    const uint32_t bv = smem_addr(smem + AttnLayout::k0 + st * 2 * kOperandBytes + kOperandBytes);
#pragma unroll
                    for (int s = 0; s < 8; ++s)
                        umma_bf16(tmem_base + 256, sw128_kmajor_desc(ap + (s >> 2) * 16384 + (s & 3) * 32),
                                  sw128_mnmajor_desc(bv + s * 2048), id_o, (j > 0 || s > 0) ? 1u : 0u);
                    umma_commit(empty + st);
                    umma_commit(ofull);
                }
                it += sg.n;
                g += sg.n;
            }
            if (!ok) attn_abort(abort_flag, p.status);
            // every MMA done before TMEM is freed (a bounded wait that an abort does not cut short)
            volatile int keep_waiting = 0;
            umma_commit(done);
            if (!mbar_wait(done, 0, &keep_waiting)) set_status(p.status, HISA_DEV_TIMEOUT);
        }
        __syncwarp();
    } else {
        // --------------------------------------------------------- softmax
        // Warps 5-12.  Warp w reads the TMEM lanes of its quadrant (heads
        // h = 32 (w mod 4) + lane) and the columns of its half (w - 5) / 4:
        // tokens 64 half .. + 63 of S and P, value dims 64 half .. + 63 of O.
        // The two halves of a head exchange their maxima (and, at the end of
        // a segment, their sums) through shared memory and a bounded barrier.
        const int quad = warp & 3;
        const int half = (warp - kWarpSoft0) >> 2;
        const int h = quad * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
        const uint32_t col0 = static_cast<uint32_t>(half * 64);
        const uint32_t p_row = smem_addr(sP);
        float* red = reinterpret_cast<float*>(smem + AttnLayout::red);     // [2][2 halves][128]
        float* lred = reinterpret_cast<float*>(smem + AttnLayout::lred);   // [2 halves][128]
        const float c2 = p.scale_log2;
        bool ok = true;
        uint32_t sc = 0, ow = 0, xn = 0, ln = 0;
        for (long long g = g0; g < g1 && ok;) {
            const Seg sg = next_seg(g, g1, T);
            int b;
            const int len_b = seq_len(p, sg.row, &b);
            float m = -INFINITY, l = 0.f;
            for (int j = 0; j < sg.n; ++j) {
                const uint32_t buf = sc & 1;
                // the tile's entries of this half, read before the wait for S
                const int base = (sg.t0 + j) * 128 + half * 64;
                const bool va = attn_valid(p, sg.row, base + lane, len_b);
                const bool vb = attn_valid(p, sg.row, base + 32 + lane, len_b);
                if (!warp_wait_a(sfull + buf, (sc >> 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t mw[2] = {__ballot_sync(0xffffffffu, va), __ballot_sync(0xffffffffu, vb)};
                const bool dense = (mw[0] & mw[1]) == 0xffffffffu;
                const uint32_t ts = tmem_base + lane_off + buf * 128 + col0;
                // pass 1: this half's maximum (raw logits; the scale is positive)
                float mx = -INFINITY;
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    float v[16];
                    tmem_ld16(ts + c * 16, v);
                    if (dense) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) mx = fmaxf(mx, v[i]);
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if ((mw[c >> 1] >> ((c & 1) * 16 + i)) & 1u) mx = fmaxf(mx, v[i]);
                    }
                }
                mx *= c2;
                // the row maximum from both halves
                const uint32_t xb = xn & 1;
                red[(xb * 2 + half) * 128 + h] = mx;
                __syncwarp();
                if (lane == 0) mbar_arrive(xbar + xb);
                if (!warp_wait_a(xbar + xb, (xn >> 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                ++xn;
                const float m_new = fmaxf(m, fmaxf(mx, red[(xb * 2 + (half ^ 1)) * 128 + h]));
                // the previous P V must be done before P is rewritten or O rescaled
                if (j > 0) {
                    if (!warp_wait_a(ofull, ow & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    ++ow;
                    tc_fence_after();
                    // the TMEM loads and stores below are warp-wide (.sync.aligned): the
                    // warp rescales together when any of its heads' maxima grew
                    const bool grew = m_new > m && m > -INFINITY;
                    if (__any_sync(0xffffffffu, grew)) {
                        const float alpha = grew ? ex2_approx(m - m_new) : 1.f;
                        l *= alpha;
                        const uint32_t to = tmem_base + lane_off + 256 + col0;
#pragma unroll 1
                        for (int c = 0; c < 4; ++c) {
                            float v[16];
                            tmem_ld16(to + c * 16, v);
                            uint32_t u[16];
#pragma unroll
                            for (int i = 0; i < 16; ++i) u[i] = __float_as_uint(v[i] * alpha);
                            tmem_st16(to + c * 16, u);
                        }
                        tmem_st_wait();
                    }
                }
                // pass 2: p = 2^(s c2 - max) in bf16 into this half of the P row, and its sum
                const bool live = m_new > -INFINITY;
                float psum = 0.f;
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    float v[16];
                    tmem_ld16(ts + c * 16, v);
                    float e[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const bool on = live && (dense || ((mw[c >> 1] >> ((c & 1) * 16 + i)) & 1u));
                        e[i] = on ? ex2_approx(fmaf(v[i], c2, -m_new)) : 0.f;
                        psum += e[i];
                    }
                    uint32_t w8[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) w8[i] = pack_bf16(e[2 * i], e[2 * i + 1]);
                    const int chunk = half * 8 + 2 * c;
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(p_row + sw128_off(h, chunk)),
                                 "r"(w8[0]), "r"(w8[1]), "r"(w8[2]), "r"(w8[3])
                                 : "memory");
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(p_row + sw128_off(h, chunk + 1)),
                                 "r"(w8[4]), "r"(w8[5]), "r"(w8[6]), "r"(w8[7])
                                 : "memory");
                }
                l += psum;
                m = m_new;
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(sempty + buf);
                ++sc;
                fence_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(pfull);
            }
            if (!ok) break;
            // the segment's last P V, then its partial result
            if (!warp_wait_a(ofull, ow & 1, abort_flag)) {
                ok = false;
                break;
            }
            ++ow;
            tc_fence_after();
            const size_t slot = static_cast<size_t>(sg.row) * T + sg.t0;
            float* po = p.part_o + (slot * 128 + h) * 128 + col0;
            const uint32_t to = tmem_base + lane_off + 256 + col0;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                float v[16];
                tmem_ld16(to + c * 16, v);
#pragma unroll
                for (int i = 0; i < 16; i += 4)
                    *reinterpret_cast<float4*>(po + c * 16 + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
            }
            // the head's sum over both halves
            lred[half * 128 + h] = l;
            __syncwarp();
            if (lane == 0) mbar_arrive(lbar);
            if (!warp_wait_a(lbar, ln & 1, abort_flag)) {
                ok = false;
                break;
            }
            ++ln;
            if (half == 0) {
                p.part_ml[slot * 256 + h] = m;
                p.part_ml[slot * 256 + 128 + h] = l + lred[128 + h];
                if (h == 0) p.seg_len[slot] = sg.n;
            }
            tc_fence_before();
            g += sg.n;
        }
        if (!ok) attn_abort(abort_flag, p.status);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMmaA) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

// One CTA per row, a thread per (head, half of the 128 dims): merges the
// row's segments (walking their lengths from tile 0) with the usual
// log-sum-exp weights, normalises, and writes o and the natural-log lse.
__global__ void __launch_bounds__(256) combine_kernel(const AttnParams p) {
    grid_dependency_wait();
    grid_launch_dependents();
    const int row = blockIdx.x;
    const int h = threadIdx.x >> 1, half = threadIdx.x & 1;
    if (h >= p.Ha) return;
    const int T = p.T;
    const size_t r0 = static_cast<size_t>(row) * T;
    float M = -INFINITY;
    for (int t = 0; t < T;) {
        const int n = p.seg_len[r0 + t];
        if (n < 1 || t + n > T) {
            set_status(p.status, HISA_DEV_TIMEOUT);
            return;
        }
        M = fmaxf(M, p.part_ml[(r0 + t) * 256 + h]);
        t += n;
    }
    float acc[64];
#pragma unroll
    for (int i = 0; i < 64; ++i) acc[i] = 0.f;
    float L = 0.f;
    for (int t = 0; t < T;) {
        const size_t slot = r0 + t;
        const float m = p.part_ml[slot * 256 + h];
        const float wgt = (M == -INFINITY) ? 0.f : exp2f(m - M);
        L += wgt * p.part_ml[slot * 256 + 128 + h];
        const float4* po = reinterpret_cast<const float4*>(p.part_o + (slot * 128 + h) * 128 + half * 64);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float4 v = po[i];
            acc[4 * i] += wgt * v.x;
            acc[4 * i + 1] += wgt * v.y;
            acc[4 * i + 2] += wgt * v.z;
            acc[4 * i + 3] += wgt * v.w;
        }
        t += p.seg_len[slot];
    }
    float4* out = reinterpret_cast<float4*>(p.out + (static_cast<size_t>(row) * p.Ha + h) * 128 + half * 64);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        float4 v;
        v.x = L > 0.f ? acc[4 * i] / L : 0.f;
        v.y = L > 0.f ? acc[4 * i + 1] / L : 0.f;
        v.z = L > 0.f ? acc[4 * i + 2] / L : 0.f;
        v.w = L > 0.f ? acc[4 * i + 3] / L : 0.f;
        out[i] = v;
    }
    if (half == 0 && p.lse)
        p.lse[static_cast<size_t>(row) * p.Ha + h] = L > 0.f ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;
}

}  // namespace

size_t attn_workspace_bytes(int n_q, int k) {
    const size_t slots = static_cast<size_t>(n_q) * ((k + 127) / 128);
    const size_t o = slots * 128 * 128 * 4, ml = slots * 256 * 4, sl = slots * 4;
    return ((o + 255) / 256 + (ml + 255) / 256 + (sl + 255) / 256) * 256;
}

void attn_carve(AttnParams& p, void* ws) {
    const size_t slots = static_cast<size_t>(p.n_q) * p.T;
    uint8_t* b = static_cast<uint8_t*>(ws);
    p.part_o = reinterpret_cast<float*>(b);
    b += (slots * 128 * 128 * 4 + 255) / 256 * 256;
    p.part_ml = reinterpret_cast<float*>(b);
    b += (slots * 256 * 4 + 255) / 256 * 256;
    p.seg_len = reinterpret_cast<int32_t*>(b);
}

cudaError_t launch_attn(const AttnParams& p, int sms, cudaStream_t s) {
    if (p.n_q <= 0) return cudaSuccess;
    const long long tiles = static_cast<long long>(p.n_q) * p.T;
    const int grid = static_cast<int>(tiles < sms ? tiles : sms);
    cudaError_t e = smem_limit(reinterpret_cast<const void*>(attn_kernel), kAttnSmem);
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kAttnThreads);
    cfg.dynamicSmemBytes = kAttnSmem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, attn_kernel, p);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t c2 = {};
    c2.gridDim = dim3(static_cast<unsigned>(p.n_q));
    c2.blockDim = dim3(256);
    c2.stream = s;
    c2.attrs = attr;
    c2.numAttrs = 1;
    e = cudaLaunchKernelEx(&c2, combine_kernel, p);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace hisa
