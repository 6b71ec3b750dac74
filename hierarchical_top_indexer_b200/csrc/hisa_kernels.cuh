// Internal interface between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <map>
#include <mutex>
#include <utility>

#include "hisa_device.cuh"

namespace hisa {

// The cache as the kernels see it (validated copy of hisa_kv).
struct KvView {
    void* keys;
    float* key_scale;
    float* pooled;
    uint16_t* pooled_hl;
    int32_t* len;
    uint32_t* status;
    int batch, cap, d, B, nblk;
    bool e4m3;
    bool pool_max;   // elementwise-max representatives (else means)
};

// What a scoring launch scores.
enum ScoreMode : int {
    kScoreBlocks = 0,   // block representatives (pooled_hl), candidates j < nb(t)
    kScoreFlat = 1,     // every key s <= t
    kScoreHisa = 2      // the keys of each row's kept blocks
};

struct ScoreParams {
    // cache
    const int32_t* len;
    const float* key_scale;
    uint32_t* status;
    int batch, cap, nblk, B;
    // query rows
    const float* w;
    const int32_t* q_seq;
    const int32_t* q_pos;
    int n_q, H, npad;
    // kept blocks (kScoreHisa input): blocks [n_q, mm], and the row plan
    // {sequence, position (-1: invalid row), kept blocks, 0} [n_q]
    const int32_t* blocks;
    const int4* plan_in;
    int mm;
    // kScoreBlocks under the units kept one level up (multi-level search):
    // block c of a row is a candidate only if unit c / bf of the level above
    // (a superblock) is in the row's parent[row, 0 .. parent_ld) (-1
    // padded); null: every block is
    const int32_t* parent;
    int parent_ld, bf;
    // with parent_n (the kept superblocks per row) the kernel loads and
    // scores only their children, bf per superblock (rows fused, bf a power
    // of two from 8 to 128, parent_ld <= 256)
    const int32_t* parent_n;
    // score keys [n_q, ldo] (order-preserving; 0 = masked slot)
    uint32_t* out;
    int ldo;
    unsigned long long* counts;   // null, or per row: representatives scored at
                                  // counts[row * counts_ld + counts_col] (blocks
                                  // mode), token slots scored one column further
    int counts_ld, counts_col;
    int tiles_per_row;            // tile slots per row (upper bound)
    long long total_tiles;        // n_q * tiles_per_row
    int stages;                   // bf16 operand stages
    int stages8;                  // e4m3 staging stages
    int nacc;                     // TMEM accumulators
    int keep_keys;                // rows share keys: keep them in L2 (else stream them)
    // e4m3 keys with d = 128 (scored on the fp8 tensor cores): per-row head
    // weights with each head's query scale folded in [n_q, npad], and whether
    // every tile's per-token scales start on a 16-byte boundary (cap % 4 == 0)
    const float* w8;
    int scale_bulk;
    // kScoreBlocks with fuse = 1: each CTA scores whole rows and keeps the own
    // block plus the best m - 1 others itself (rows of at most kFuseMaxBlocks
    // blocks); outputs as the block selection's
    int fuse, m;
    int32_t* sel_blocks;          // [n_q, mm]
    int32_t* sel_nblocks;         // [n_q]
    int4* sel_plan;               // [n_q]
    int32_t* sel_blocks_out;      // [n_q, mm] or null
    int32_t* sel_nblocks_out;     // [n_q] or null
    // kScoreBlocks in the decode step (app = 1, fuse = 1): row b is sequence
    // b, whose new key the append kernel launched just before is writing at
    // position len[b] (concurrently: it only changes the representative of
    // the row's own block, which is kept whatever its score); the row selects
    // for position len[b] (cap - 1 for a full sequence, which appends
    // nothing), and after waiting for the append the kernel advances len[b]
    int app;
    int32_t* len_w;               // the cache's lengths (app = 1)
    // kScoreBlocks over one context-parallel shard (cp = 1): the cache holds
    // the global positions [tok_off, tok_off + cap) of every sequence, q_pos
    // are global positions, and a row's candidates are the shard's blocks
    // that cp_visible_blocks admits
    int cp, tok_off;
};

constexpr int kFuseMaxBlocks = 512;
constexpr int kParentBits = 32768;    // superblocks a kept-superblock mask can cover

enum SelectMode : int {
    kSelBlocks = 0,      // keep own block + best m-1 others -> blocks list
    kSelHisaTokens = 1,  // keep top-k of the kept blocks' token slots
    kSelFlatTokens = 2,  // keep top-k of keys 0..t
    kSelF32Rows = 3,     // keep top-k of n given fp32 values per row
    kSelCpBlocks = 4,    // one shard's block candidates: best m-1 visible blocks
                         // but the own one, then the own block (score +inf)
    kSelMerge = 5        // top-k of `lists` (id, score) lists per row
};

// Rows of up to kRowKeys slots are selected by one CTA (the context-parallel
// modes only ever take that path).
constexpr int kRowKeys = 24576;

// Context parallelism: a shard holds the global positions [tok_off, tok_off +
// cap) of every sequence (tok_off and cap multiples of B).  For the query row
// i at global position q_pos[i], returns how many of the shard's blocks it
// sees (0: its prefix ends before the shard), with *own = 1 when the shard
// holds the query position (the last visible block is then the row's own
// block) and *tl = q_pos - tok_off; -1 for an invalid row (bad sequence, a
// negative position, or a position past the sequence's end).
__device__ __forceinline__ int cp_visible_blocks(const int32_t* q_seq, const int32_t* q_pos,
                                                 const int32_t* len, int batch, int cap, int B,
                                                 int tok_off, int i, int* seq_out, int* own, int* tl) {
    const int b = q_seq[i];
    *seq_out = b;
    *own = 0;
    *tl = -1;
    if (b < 0 || b >= batch) return -1;
    const int n = len[b];
    const int t = q_pos[i];
    if (n < 0 || n > cap || t < 0) return -1;
    const long long l = static_cast<long long>(t) - tok_off;
    if (l < 0) return 0;
    *tl = static_cast<int>(l);
    if (l < n) {
        *own = 1;
        return static_cast<int>(l) / B + 1;
    }
    return n == cap ? cap / B : -1;   // a full shard is wholly visible
}


struct SelectParams {
    int mode;
    const uint32_t* keys;   // [rows, ldk] score keys (modes 0-2)
    const float* x;         // [rows, n] fp32 (mode 3)
    int ldk, n;
    int rows, k;
    // query rows (modes 0-2)
    const int32_t* len;
    const int32_t* q_seq;
    const int32_t* q_pos;
    uint32_t* status;
    int batch, cap, B, m, mm;
    // kept blocks: written by mode 0, read by mode 1
    int32_t* blocks;
    int32_t* nblocks;
    int4* plan;              // {sequence, position or -1, kept blocks, 0} per row
    // outputs
    int32_t* idx;       // [rows, k]   (modes 1-3)
    float* scores;      // [rows, k] or null
    int32_t* blocks_out;     // [rows, mm] or null (mode 0 copy for inspection)
    int32_t* nblocks_out;    // [rows] or null
    int tree;                // mode 0 over masked candidates: no keep-everything shortcut
    int id_off;              // added to every emitted id (modes 1, 4: a shard's first
                             // token / block); mode 4 also reads tok_off = id_off * B
    // mode 5: ids [lists, rows, n] (-1: empty) and their scores x [lists, rows, n];
    // the concatenated lists of a row must ascend in id
    const int32_t* ids;
    int lists;
};

// Context-parallel token plan: from each row's merged global block list
// kept [rows, m] (ascending, -1 padded), the visible blocks of the shard at
// tok_off, as local ids into blocks [rows, mm] with counts nblocks and plans
// {sequence, position for the token masks, count, 0}.  A valid row always
// has its own block (global id q_pos / B) among the kept ones; a row without
// it is invalid on every shard (plan position -1, HISA_DEV_BAD_QUERY).
struct CpLocalizeParams {
    const int32_t* kept;
    int m;
    const int32_t* q_seq;
    const int32_t* q_pos;
    const int32_t* len;
    uint32_t* status;
    int batch, cap, B, tok_off, rows, mm;
    int32_t* blocks;
    int32_t* nblocks;
    int4* plan;
};
cudaError_t launch_cp_localize(const CpLocalizeParams& p, cudaStream_t s);

// Sparse attention over selected tokens (attn.cu): Ha <= 128 query heads of
// d = 128 sharing one key and one value head, k selected entries per row.
struct AttnParams {
    const uint16_t* q;       // [n_q, Ha, 128] bf16
    const uint16_t* kc;      // [batch, cap, 128] bf16
    const uint16_t* vc;      // [batch, cap, 128] bf16
    const int32_t* idx;      // [n_q, k]
    const int32_t* q_seq;    // [n_q]
    const int32_t* len;      // [batch]
    int batch, cap, n_q, Ha, k, T;   // T = tiles of 128 entries per row
    float scale_log2;        // softmax scale * log2(e)
    float* part_o;           // workspace: [n_q * T, 128, 128] unnormalised segment outputs
    float* part_ml;          // workspace: [n_q * T, 2, 128] segment max (log2 domain), sum
    int32_t* seg_len;        // workspace: [n_q * T] tiles of the segment starting there
    float* out;              // [n_q, Ha, 128]
    float* lse;              // [n_q, Ha] or null
    uint32_t* status;
};
size_t attn_workspace_bytes(int n_q, int k);
void attn_carve(AttnParams& p, void* ws);
cudaError_t launch_attn(const AttnParams& p, int sms, cudaStream_t s);

// One warp waiting on an mbarrier that never completes (diag.cu).
cudaError_t launch_wait_probe(uint32_t* status, cudaStream_t s);

// Raise a kernel's dynamic shared-memory limit to at least `bytes` on the
// current device, once: the attribute call costs microseconds of host time,
// so it is made only the first time a kernel needs a larger limit there.
// (A cudaDeviceReset discards the attribute but not this record; a process
// that resets a device it keeps using would see the next large launch fail
// with an invalid-value error.)
inline cudaError_t smem_limit(const void* fn, size_t bytes) {
    static std::mutex mu;
    static std::map<std::pair<const void*, int>, size_t> have;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    {
        std::lock_guard<std::mutex> g(mu);
        const auto it = have.find({fn, dev});
        if (it != have.end() && it->second >= bytes) return cudaSuccess;
    }
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> g(mu);
    size_t& h = have[{fn, dev}];
    if (h < bytes) h = bytes;
    return cudaSuccess;
}

cudaError_t launch_pool(const KvView& kv, cudaStream_t s);
// step = true: the decode step's append, which leaves len to the scoring
// kernel that follows it (see append_kernel).
cudaError_t launch_append(const KvView& kv, const void* tok, const float* tok_scale,
                          cudaStream_t s, bool step = false);
// Re-pool each sequence's trailing block (the one holding key len - 1).
cudaError_t launch_pool_tail(const KvView& kv, cudaStream_t s);

// Scoring: tensor maps built by the caller.  `keys_map` covers keys
// ([batch*cap, d], bf16 swizzled 128B boxes, or e4m3 plain boxes) or, for
// kScoreBlocks, pooled_hl ([batch*nblk, 2d] bf16).
int score_config(int mode, bool e4m3, int d, int npad, int* stages, int* stages8, int* nacc);
size_t score_smem_bytes(int mode, bool e4m3, int d, int npad, int stages, int stages8);
cudaError_t launch_score(int mode, bool e4m3, int d, const CUtensorMap& keys_map,
                         const CUtensorMap& q_map, const ScoreParams& p, int grid,
                         cudaStream_t s);

cudaError_t launch_select(const SelectParams& p, int max_n, int sms, cudaStream_t s);

// Block-centric token scoring (score_bc.cu) for rows sharing their keys:
// bf16 keys, B = 128, npad in {32, 64, 128}, H % 4 == 0, kept lists of at
// most 2048 blocks.  Output: score keys [n_q, ldo] as kScoreHisa writes them.
struct BcParams {
    const int4* plan;        // [n_q] {sequence, position (-1: invalid), kept blocks, 0}
    const float* w;          // [n_q, H]
    int n_q, H, npad, cap, nblk, mm;
    // inverted index of the kept lists (workspace), built by launch_bc_index
    int32_t* cnt;            // [batch * nblk] pairs per block
    int32_t* off;            // [batch * nblk] first pair of each block
    int32_t* rank;           // [n_q * mm] a pair's place in its block's list
    uint32_t* pairs_w;       // [n_q * mm] (row << 11) | r, grouped by block
    int4* units_w;           // [bc_max_units] {b * nblk + j, first pair, pairs, 0}
    int32_t* n_units_w;      // [1]
    const uint32_t* pairs;   // read views of the three above
    const int4* units;
    const int32_t* n_units;
    uint32_t* out;           // [n_q, ldo] score keys
    int ldo;
    uint32_t* status;
    unsigned long long* counts;   // null, or the token slots scored per row go to
    int counts_ld, counts_col;    // counts[row * counts_ld + counts_col + 1]
};
size_t bc_max_units(int n_q, int mm, int nbj);
cudaError_t launch_bc_index(const BcParams& p, const int32_t* blocks, int nbj, cudaStream_t s);
cudaError_t launch_bc_score(const CUtensorMap& kmap, const CUtensorMap& qmap, const BcParams& p, int sms,
                            cudaStream_t s);

// Query heads for scoring e4m3 keys (d = 128) on the fp8 tensor cores: every
// head of Q [n_q, H, 128] bf16 is scaled by a power of two 2^e and split into
// two e4m3 pieces, q * 2^e = q1 + q2; q8 [n_q, 2 * npad, 128] holds the q1
// rows then the q2 rows (zero rows pad H to npad); w8 [n_q, npad] = w * 2^-e.
cudaError_t launch_qsplit(const uint16_t* Q, const float* w, int n_q, int H, int npad, uint8_t* q8,
                          float* w8, cudaStream_t s);

}  // namespace hisa
