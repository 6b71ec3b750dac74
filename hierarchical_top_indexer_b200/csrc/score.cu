// Indexer scoring on the tcgen05 tensor cores.
//
// One kernel scores 128 candidates per tile for one query row:
//     score(i, x) = sum_h w[i,h] * max(0, q[i,h,:] . x)
// (the lightning-indexer form HISA reuses for both stages: gptget.net
// summary, "Methodology" — block representatives and candidate tokens are
// scored by the same original indexer).  The dot products are one UMMA per
// 16-wide K step with the candidates as M (128 rows) and the H heads (padded
// to a multiple of 16) as N, so that each TMEM lane ends up holding one
// candidate's H head logits; the ReLU, the head weights and the head sum run
// in the epilogue on that one thread's registers.
//
// Candidates come in three forms:
//   kScoreBlocks  block representatives: pooled_hl rows (bf16 hi and lo of
//                 the fp32 mean, two accumulating UMMAs per K step);
//   kScoreFlat    every key s <= t (the flat scan);
//   kScoreHisa    the keys of the row's kept blocks (gathered block-wise by
//                 TMA: a kept block is one or more contiguous tile rows).
// e4m3 keys are staged as bytes, widened to bf16 in shared memory by four
// converter warps (exact), and their per-token scale multiplies the score
// (ReLU(s*x) = s*ReLU(x) for s > 0).
//
// Warp roles (persistent, one CTA per SM, contiguous range of tiles):
//   warp 0       TMA producer (keys / representatives, query heads)
//   warp 1       TMEM owner and UMMA issuer
//   warps 2-5    epilogue (TMEM -> registers -> score key -> global)
//   warps 6-9    e4m3 -> bf16 converters (e4m3 keys only)
// Every mbarrier wait is bounded; on expiry the CTA raises HISA_DEV_TIMEOUT,
// drains its outstanding copies and returns.
#include "hisa_kernels.cuh"

namespace hisa {

namespace {

constexpr int kTileRows = 128;
constexpr int kHalfBytes = kTileRows * 128;   // one 128-byte-wide K slab of a tile
constexpr int kWarpProducer = 0;
constexpr int kWarpMma = 1;
constexpr int kWarpEpi0 = 2;
constexpr int kWarpConv0 = 6;
constexpr int kMinSmem = 120 * 1024;          // keeps one CTA (and its TMEM) per SM
constexpr int kMaxSmem = 232448;

struct Layout {
    uint32_t a, s8, q, w, bars, misc, total;
};

__host__ __device__ inline Layout score_layout(int mode, bool e4m3, int d, int npad, int stages) {
    const int halves = d / 64;
    const int stage = (mode == kScoreBlocks ? 2 : 1) * halves * kHalfBytes;
    const int stage8 = e4m3 ? kTileRows * d : 0;
    Layout L;
    uint32_t off = 0;
    L.a = off;
    off += stages * stage;
    L.s8 = off;
    off += stages * stage8;
    L.q = off;
    off += 2 * halves * npad * 128;
    L.w = off;
    off += 4 * 128 * 4;                      // one 128-float weight slot per epilogue warp
    L.bars = off;
    off += (4 * stages + 8) * 8;
    L.misc = off;
    off += 16;
    L.total = off;
    return L;
}

__host__ __device__ inline uint32_t tmem_columns(int npad) {
    uint32_t c = 32;
    while (c < static_cast<uint32_t>(2 * npad)) c <<= 1;
    return c;
}

struct Tile {
    int row, ti, b, t, lim;
};

// Next tile of [g, g1) that holds at least one candidate.  All roles walk the
// same sequence, so they agree on tile order without exchanging metadata.
template <int MODE>
__device__ __forceinline__ bool next_tile(const ScoreParams& p, long long& g, long long g1,
                                          Tile& T) {
    while (g < g1) {
        const long long cur = g++;
        const int row = static_cast<int>(cur / p.tiles_per_row);
        const int ti = static_cast<int>(cur % p.tiles_per_row);
        int b;
        const int t = query_position(p.q_seq, p.q_pos, p.len, p.batch, p.cap, row, &b);
        if (t < 0) continue;
        int lim;
        if (MODE == kScoreBlocks) lim = t / p.B + 1;          // visible blocks
        else if (MODE == kScoreFlat) lim = t + 1;             // visible keys
        else lim = p.nblocks[row] * p.B;                      // kept token slots
        if (ti * kTileRows >= lim) continue;
        T.row = row;
        T.ti = ti;
        T.b = b;
        T.t = t;
        T.lim = lim;
        return true;
    }
    return false;
}

__device__ __forceinline__ void raise_abort(volatile int* abort_flag, uint32_t* status) {
    *abort_flag = 1;
    set_status(status, HISA_DEV_TIMEOUT);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

// Eight e4m3 codes -> eight bf16 (exact: every e4m3 value is a bf16 value).
__device__ __forceinline__ uint4 e4m3x8_to_bf16x8(uint2 raw) {
    const uint32_t w[2] = {raw.x, raw.y};
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        const __nv_fp8x2_storage_t lo = static_cast<__nv_fp8x2_storage_t>(w[q] & 0xFFFFu);
        const __nv_fp8x2_storage_t hi = static_cast<__nv_fp8x2_storage_t>(w[q] >> 16);
        const float2 a = __half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2(lo, __NV_E4M3)));
        const float2 b = __half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2(hi, __NV_E4M3)));
        o[2 * q] = pack_bf16x2(a.x, a.y);
        o[2 * q + 1] = pack_bf16x2(b.x, b.y);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

template <int MODE, bool E4M3, int D>
__global__ void __launch_bounds__(E4M3 ? 320 : 192, 1)
    score_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap qmap,
                 const ScoreParams p) {
    constexpr int kHalves = D / 64;
    constexpr int kOps = (MODE == kScoreBlocks) ? 2 : 1;
    constexpr int kStageBytes = kOps * kHalves * kHalfBytes;
    constexpr int kStage8Bytes = kTileRows * D;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const Layout L = score_layout(MODE, E4M3, D, p.npad, p.stages);
    const int S = p.stages;
    uint8_t* sA = smem + L.a;
    uint8_t* s8 = smem + L.s8;
    uint8_t* sQ = smem + L.q;
    float* sW = reinterpret_cast<float*>(smem + L.w);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint64_t* full = bars;             // stage holds bf16 operands (TMA or converters)
    uint64_t* empty = bars + S;        // stage free again (UMMA done reading)
    uint64_t* sfull = bars + 2 * S;    // e4m3 staging landed
    uint64_t* sempty = bars + 3 * S;   // e4m3 staging converted
    uint64_t* tfull = bars + 4 * S;    // accumulator ready   [2]
    uint64_t* tempty = tfull + 2;      // accumulator drained [2]
    uint64_t* qfull = tfull + 4;       // query heads landed  [2]
    uint64_t* qempty = tfull + 6;      // query heads free    [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.misc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.misc + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int npad = p.npad;
    const uint32_t ncols = tmem_columns(npad);
    const int q_slot_bytes = kHalves * npad * 128;

    if (warp == kWarpProducer && lane == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full + s, E4M3 ? 4 : 1);
            mbar_init(empty + s, 1);
            mbar_init(sfull + s, 1);
            mbar_init(sempty + s, 4);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull + a, 1);
            mbar_init(tempty + a, 4);
            mbar_init(qfull + a, 1);
            mbar_init(qempty + a, 1);
        }
        *abort_flag = 0;
        fence_barrier_init();
        fence_async_smem();
        tma_prefetch_desc(&amap);
        tma_prefetch_desc(&qmap);
    }
    if (warp == kWarpMma) {
        tmem_alloc(tmem_slot, ncols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const long long g0 = p.total_tiles * blockIdx.x / gridDim.x;
    const long long g1 = p.total_tiles * (blockIdx.x + 1) / gridDim.x;
    const int BR = (MODE == kScoreBlocks) ? kTileRows : (p.B < kTileRows ? p.B : kTileRows);

    if (warp == kWarpProducer) {
        if (lane == 0) {
            const uint64_t pol = policy_evict_first();
            long long g = g0;
            Tile T;
            int it = 0, qloads = 0, cur_row = -1;
            bool ok = true;
            while (next_tile<MODE>(p, g, g1, T)) {
                if (T.row != cur_row) {
                    const int qs = qloads & 1;
                    if (qloads >= 2 && !mbar_wait(qempty + qs, ((qloads - 2) >> 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(qfull + qs, q_slot_bytes);
#pragma unroll
                    for (int kh = 0; kh < kHalves; ++kh)
                        tma_load_2d(sQ + qs * q_slot_bytes + kh * npad * 128, &qmap, qfull + qs,
                                    kh * 64, T.row * p.H);
                    ++qloads;
                    cur_row = T.row;
                }
                const int s = it % S;
                const uint32_t ph = (it / S) & 1;
                uint64_t* fb = E4M3 ? sfull + s : full + s;
                uint64_t* eb = E4M3 ? sempty + s : empty + s;
                if (!mbar_wait(eb, ph ^ 1, abort_flag)) {
                    ok = false;
                    break;
                }
                if (MODE == kScoreBlocks) {
                    mbar_arrive_expect_tx(fb, kStageBytes);
                    const int row0 = T.b * p.nblk + T.ti * kTileRows;
#pragma unroll
                    for (int op = 0; op < 2; ++op)
#pragma unroll
                        for (int kh = 0; kh < kHalves; ++kh)
                            tma_load_2d(sA + s * kStageBytes + (op * kHalves + kh) * kHalfBytes, &amap,
                                        fb, op * D + kh * 64, row0);
                } else {
                    mbar_arrive_expect_tx(fb, E4M3 ? kStage8Bytes : kStageBytes);
                    for (int sub = 0; sub < kTileRows / BR; ++sub) {
                        int srow;
                        if (MODE == kScoreFlat) {
                            srow = T.b * p.cap + T.ti * kTileRows + sub * BR;
                        } else {
                            const int slot = T.ti * kTileRows + sub * BR;
                            const int r = slot / p.B, off = slot % p.B;
                            const int blk = slot < T.lim ? p.blocks[T.row * p.mm + r] : 0;
                            srow = T.b * p.cap + blk * p.B + off;
                        }
                        if (E4M3) {
                            tma_load_2d_hint(s8 + s * kStage8Bytes + sub * BR * D, &amap, fb, 0, srow,
                                             pol);
                        } else {
#pragma unroll
                            for (int kh = 0; kh < kHalves; ++kh)
                                tma_load_2d_hint(sA + s * kStageBytes + kh * kHalfBytes + sub * BR * 128,
                                                 &amap, fb, kh * 64, srow, pol);
                        }
                    }
                }
                ++it;
            }
            if (!ok) raise_abort(abort_flag, p.status);
            // Drain: no copy into, and no arrive on, this CTA's shared memory
            // may still be pending when it exits.
            for (int n = it > S ? it - S : 0; n < it; ++n) {
                const int s = n % S;
                const uint32_t ph = (n / S) & 1;
                if (ok) mbar_wait(E4M3 ? sempty + s : empty + s, ph, nullptr);
                else mbar_wait(E4M3 ? sfull + s : full + s, ph, nullptr);
            }
            if (qloads >= 1) {
                if (ok && qloads >= 2)
                    mbar_wait(qempty + ((qloads - 2) & 1), ((qloads - 2) >> 1) & 1, nullptr);
                if (!ok) mbar_wait(qfull + ((qloads - 1) & 1), ((qloads - 1) >> 1) & 1, nullptr);
            }
        }
    } else if (warp == kWarpMma) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(static_cast<uint32_t>(npad));
            long long g = g0;
            Tile T;
            int it = 0, qloads = 0, cur_row = -1;
            bool ok = true;
            while (next_tile<MODE>(p, g, g1, T)) {
                if (T.row != cur_row) {
                    if (qloads > 0) umma_commit(qempty + ((qloads - 1) & 1));
                    if (!mbar_wait(qfull + (qloads & 1), (qloads >> 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    ++qloads;
                    cur_row = T.row;
                }
                const int s = it % S;
                const int a = it & 1;
                if (!mbar_wait(full + s, (it / S) & 1, abort_flag) ||
                    !mbar_wait(tempty + a, ((it >> 1) & 1) ^ 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(a * npad);
                const uint32_t a_base = smem_addr(sA + s * kStageBytes);
                const uint32_t q_base = smem_addr(sQ + ((qloads - 1) & 1) * q_slot_bytes);
#pragma unroll
                for (int kh = 0; kh < kHalves; ++kh) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t bdesc = sw128_kmajor_desc(q_base + kh * npad * 128 + kk * 32);
                        const uint64_t adesc = sw128_kmajor_desc(a_base + kh * kHalfBytes + kk * 32);
                        umma_bf16(d_tmem, adesc, bdesc, idesc, (kh | kk) ? 1u : 0u);
                        if (MODE == kScoreBlocks) {
                            const uint64_t ldesc =
                                sw128_kmajor_desc(a_base + (kHalves + kh) * kHalfBytes + kk * 32);
                            umma_bf16(d_tmem, ldesc, bdesc, idesc, 1u);
                        }
                    }
                }
                umma_commit(empty + s);
                umma_commit(tfull + a);
                ++it;
            }
            if (!ok) raise_abort(abort_flag, p.status);
            // every UMMA of this CTA has finished before TMEM is released
            if (it > 0) mbar_wait(tfull + ((it - 1) & 1), ((it - 1) >> 1) & 1, nullptr);
        }
    } else if (warp >= kWarpEpi0 && warp < kWarpEpi0 + 4) {
        const int quad = warp & 3;             // TMEM lanes this warp may read
        const int r = quad * 32 + lane;        // tile row = candidate
        float* wv = sW + (warp - kWarpEpi0) * 128;
        long long g = g0;
        Tile T;
        int it = 0, cur_row = -1;
        while (next_tile<MODE>(p, g, g1, T)) {
            if (T.row != cur_row) {
                __syncwarp();
                for (int h = lane; h < 128; h += 32) wv[h] = h < p.H ? p.w[T.row * p.H + h] : 0.f;
                __syncwarp();
                cur_row = T.row;
            }
            const int a = it & 1;
            if (!mbar_wait(tfull + a, (it >> 1) & 1, abort_flag)) {
                raise_abort(abort_flag, p.status);
                break;
            }
            tc_fence_after();
            const uint32_t taddr =
                tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(a * npad);
            float acc = 0.f;
            for (int c = 0; c < npad; c += 16) {
                float v[16];
                tmem_ld16(taddr + c, v);
                tmem_ld_wait();
#pragma unroll
                for (int h = 0; h < 16; ++h)
                    if (c + h < p.H) acc = fmaf(wv[c + h], fmaxf(v[h], 0.f), acc);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty + a);

            uint32_t* out = p.out + static_cast<size_t>(T.row) * p.ldo;
            if (MODE == kScoreBlocks) {
                const int j = T.ti * kTileRows + r;
                const bool valid = j < T.lim;
                out[j] = valid ? score_key(acc) : 0u;
                if (p.counts) {
                    const int n = __popc(__ballot_sync(0xffffffffu, valid));
                    if (lane == 0 && n) atomicAdd(p.counts + 2 * T.row, static_cast<unsigned long long>(n));
                }
            } else {
                const int c = T.ti * kTileRows + r;
                int s;
                bool valid;
                if (MODE == kScoreFlat) {
                    s = c;
                    valid = s <= T.t;
                } else {
                    const bool slot_ok = c < T.lim;
                    const int blk = slot_ok ? p.blocks[T.row * p.mm + c / p.B] : 0;
                    s = blk * p.B + c % p.B;
                    valid = slot_ok && s <= T.t;
                    if (p.counts) {
                        const int n = __popc(__ballot_sync(0xffffffffu, slot_ok));
                        if (lane == 0 && n)
                            atomicAdd(p.counts + 2 * T.row + 1, static_cast<unsigned long long>(n));
                    }
                }
                if (E4M3 && valid) acc *= p.key_scale[static_cast<size_t>(T.b) * p.cap + s];
                out[c] = valid ? score_key(acc) : 0u;
            }
            ++it;
        }
    } else if (E4M3 && warp >= kWarpConv0) {
        const int cw = warp - kWarpConv0;
        long long g = g0;
        Tile T;
        int it = 0;
        bool ok = true;
        while (next_tile<MODE>(p, g, g1, T)) {
            const int s = it % S;
            const uint32_t ph = (it / S) & 1;
            if (!mbar_wait(sfull + s, ph, abort_flag) || !mbar_wait(empty + s, ph ^ 1, abort_flag)) {
                ok = false;
                break;
            }
            const uint8_t* src = s8 + s * kStage8Bytes;
            uint8_t* dst = sA + s * kStageBytes;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int rr = cw * 32 + i * 4 + (lane >> 3);
                const int cc = lane & 7;
#pragma unroll
                for (int kh = 0; kh < kHalves; ++kh) {
                    const uint2 raw = *reinterpret_cast<const uint2*>(src + rr * D + kh * 64 + cc * 8);
                    *reinterpret_cast<uint4*>(dst + kh * kHalfBytes + rr * 128 + ((cc ^ (rr & 7)) << 4)) =
                        e4m3x8_to_bf16x8(raw);
                }
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(full + s);
                mbar_arrive(sempty + s);
            }
            ++it;
        }
        if (!ok) raise_abort(abort_flag, p.status);
        if (ok && cw == 0 && lane == 0)
            for (int n = it > S ? it - S : 0; n < it; ++n) mbar_wait(empty + n % S, (n / S) & 1, nullptr);
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpMma) tmem_dealloc(tmem_base, ncols);
}

template <int MODE, bool E4M3, int D>
cudaError_t launch_t(const CUtensorMap& amap, const CUtensorMap& qmap, const ScoreParams& p, int grid,
                     cudaStream_t s) {
    const size_t smem = score_smem_bytes(MODE, E4M3, D, p.npad, p.stages);
    auto* fn = score_kernel<MODE, E4M3, D>;
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    fn<<<grid, E4M3 ? 320 : 192, smem, s>>>(amap, qmap, p);
    return cudaGetLastError();
}

}  // namespace

size_t score_smem_bytes(int mode, bool e4m3, int d, int npad, int stages) {
    const size_t need = score_layout(mode, e4m3, d, npad, stages).total + 1024;
    return need < static_cast<size_t>(kMinSmem) ? static_cast<size_t>(kMinSmem) : need;
}

int score_stages(int mode, bool e4m3, int d, int npad) {
    int best = 0;
    for (int s = 2; s <= 8; ++s)
        if (score_layout(mode, e4m3, d, npad, s).total + 1024 <= static_cast<uint32_t>(kMaxSmem)) best = s;
    return best;
}

cudaError_t launch_score(int mode, bool e4m3, int d, const CUtensorMap& amap, const CUtensorMap& qmap,
                         const ScoreParams& p, int grid, cudaStream_t s) {
    if (mode == kScoreBlocks)
        return d == 128 ? launch_t<kScoreBlocks, false, 128>(amap, qmap, p, grid, s)
                        : launch_t<kScoreBlocks, false, 64>(amap, qmap, p, grid, s);
    if (mode == kScoreFlat) {
        if (e4m3)
            return d == 128 ? launch_t<kScoreFlat, true, 128>(amap, qmap, p, grid, s)
                            : launch_t<kScoreFlat, true, 64>(amap, qmap, p, grid, s);
        return d == 128 ? launch_t<kScoreFlat, false, 128>(amap, qmap, p, grid, s)
                        : launch_t<kScoreFlat, false, 64>(amap, qmap, p, grid, s);
    }
    if (e4m3)
        return d == 128 ? launch_t<kScoreHisa, true, 128>(amap, qmap, p, grid, s)
                        : launch_t<kScoreHisa, true, 64>(amap, qmap, p, grid, s);
    return d == 128 ? launch_t<kScoreHisa, false, 128>(amap, qmap, p, grid, s)
                    : launch_t<kScoreHisa, false, 64>(amap, qmap, p, grid, s);
}

}  // namespace hisa
