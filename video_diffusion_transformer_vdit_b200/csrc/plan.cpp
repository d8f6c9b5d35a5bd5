// Host side of libvdit: error reporting, geometry checks and the tile schedule (vdit_attn_plan).
//
// The schedule lists, per 128-query tile, the 128-key tiles holding at least one kept pair of the
// block-causal / radial mask ("DynamicRad: Content-Adaptive Sparse Attention for Long Video
// Diffusion", section 2; Wave Forcing / WaveRT news item: block-causal chunks), each flagged full
// when complete and wholly kept. It is derived without touching individual pairs: a tile's token
// range splits into row segments (constant frame and patch row h, a contiguous run of columns w),
// and for two segments every predicate term is either constant (validity, causal chunk order,
// |dt|, |dh|) or a function of |w_q - w_k| over two integer intervals, whose minimum and maximum
// are closed forms. Cost is O(tiles x segment pairs) instead of O(tokens^2). The query tiles are
// computed independently by a few host threads and merged in tile order, so the plan (the
// numbering of its shared keep-mask blocks included) does not depend on the thread count.
#include <algorithm>
#include <atomic>
#include <climits>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <functional>
#include <new>
#include <unordered_map>
#include <thread>
#include <vector>

#include <cuda_runtime.h>

#include "internal.h"

namespace {
thread_local std::string g_last_error;
}

namespace vdit {

int fail(int code, const std::string& msg) {
    g_last_error = msg;
    return code;
}

int cuda_check(int err, const char* what) {
    if (err == 0) return VDIT_OK;
    return fail(VDIT_ERR_CUDA, std::string(what) + ": " +
                                   cudaGetErrorString(static_cast<cudaError_t>(err)));
}

int check_geom(const vdit_geom* g) {
    if (!g) return fail(VDIT_ERR_INVALID_ARG, "geometry is NULL");
    if (g->grid_h < 1 || g->grid_w < 1 || g->grid_h > VDIT_MAX_GRID || g->grid_w > VDIT_MAX_GRID)
        return fail(VDIT_ERR_INVALID_ARG, "grid_h/grid_w must be in [1, VDIT_MAX_GRID]");
    if (g->heads < 1) return fail(VDIT_ERR_INVALID_ARG, "heads must be >= 1");
    if (g->head_dim != 64 && g->head_dim != 128)
        return fail(VDIT_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
    if (g->band_t <= 0 || g->band_h <= 0 || g->band_w <= 0 || (g->band_t | g->band_h | g->band_w) & 1)
        return fail(VDIT_ERR_INVALID_ARG, "RoPE bands must be positive and even");
    if (g->band_t + g->band_h + g->band_w != g->head_dim)
        return fail(VDIT_ERR_INVALID_ARG, "RoPE bands must sum to head_dim");
    if (!(g->theta > 1.0)) return fail(VDIT_ERR_INVALID_ARG, "theta must be > 1");
    long long ft = (long long)g->grid_h * g->grid_w;
    if (ft * (VDIT_MAX_FRAME + 1) > INT_MAX / 2)
        return fail(VDIT_ERR_UNSUPPORTED, "frame too large");
    return VDIT_OK;
}

}  // namespace vdit

extern "C" const char* vdit_last_error(void) { return g_last_error.c_str(); }

namespace {

struct Seg {
    int t;      // global frame (queries) or held frame (keys); -1 = empty slot
    int h;      // patch row
    int wlo, whi;  // inclusive column range
    int off;    // offset of the segment's first token from the start of the split range
};

// Splits tokens [lo, hi) of a frame-major (frame, h, w) sequence into row segments. frame_of maps
// the local frame index (queries) or the frame slot (keys) to a global frame.
template <class F>
void segments(int lo, int hi, int grid_h, int grid_w, F frame_of, std::vector<Seg>& out) {
    out.clear();
    const int ft = grid_h * grid_w;
    int tok = lo;
    while (tok < hi) {
        const int f = tok / ft, rem = tok % ft, h = rem / grid_w, w = rem % grid_w;
        const int run = std::min(hi - tok, grid_w - w);
        out.push_back(Seg{frame_of(f), h, w, w + run - 1, tok - lo});
        tok += run;
    }
}

// Radius of the radial window at temporal distance dt: the largest Chebyshev distance d with
// d <= w0 * 2^(-gamma_shift * dt), i.e. floor(w0 / 2^s), s = gamma_shift * dt; INT_MAX when
// the whole frame is kept (long-range frame, or no radial term).
int radius_at(const vdit_mask& m, int dt) {
    if (!(m.kind & VDIT_MASK_RADIAL)) return INT_MAX;
    if (m.lambda > 0 && dt % m.lambda == 0) return INT_MAX;
    const long long s = (long long)m.gamma_shift * dt;
    const long long r = s >= 63 ? 0 : (m.w0 >> s);
    return r > INT_MAX ? INT_MAX : (int)r;
}

// Number of (a, b) in [a0, a1] x [b0, b1] with |a - b| <= r.
long long pairs_within(int a0, int a1, int b0, int b1, int r) {
    if (r == INT_MAX) return (long long)(a1 - a0 + 1) * (b1 - b0 + 1);
    long long n = 0;
    for (int a = a0; a <= a1; ++a) {
        const long long lo = std::max<long long>(b0, (long long)a - r);
        const long long hi = std::min<long long>(b1, (long long)a + r);
        if (hi >= lo) n += hi - lo + 1;
    }
    return n;
}

// Appends the keep mask of one partial tile: its query row segments `qs` (rows q0 .. of the tile,
// segment offsets relative to q0) against the key tile whose row segments are `keys`; 128 rows x
// 4 words, bit k of row r set iff key k is kept for query q0 + r. The predicate's frame and row
// terms are constant on a (query segment, key segment) pair, so they are evaluated once per pair;
// per query row the kept keys of a key segment are then one run of columns (the Chebyshev window
// is an interval of w). Key segments at a frame offset (key frame - query frame) listed in
// skip_dt are left out.
void tile_mask(const vdit_plan& p, const std::vector<Seg>& qs, const std::vector<Seg>& keys,
               std::vector<uint32_t>& out, const std::vector<int>* skip_dt = nullptr) {
    const size_t base = out.size();
    out.resize(base + 512, 0u);
    uint32_t* blk = out.data() + base;
    const bool causal = p.m.kind & VDIT_MASK_BLOCK_CAUSAL;
    for (const Seg& a : qs) {
        for (const Seg& b : keys) {
            if (b.t < 0) continue;
            if (skip_dt && std::find(skip_dt->begin(), skip_dt->end(), b.t - a.t) != skip_dt->end()) continue;
            if (causal && b.t / p.m.chunk_frames > a.t / p.m.chunk_frames) continue;
            const long long rad = p.radius[std::abs(a.t - b.t)];
            if (std::abs(a.h - b.h) > rad) continue;
            for (int wq = a.wlo; wq <= a.whi; ++wq) {
                const long long lo = std::max<long long>(b.wlo, wq - rad);
                const long long hi = std::min<long long>(b.whi, wq + rad);
                if (lo > hi) continue;
                // keys k0 .. k1 of the tile as a 128-bit run, OR-ed into the row's four words
                const int k0 = b.off + (int)(lo - b.wlo), k1 = b.off + (int)(hi - b.wlo);
                const unsigned __int128 one = 1;
                const unsigned __int128 run = (k1 == 127 ? ~(unsigned __int128)0 : (one << (k1 + 1)) - 1) &
                                              ~((one << k0) - 1);
                uint32_t* row = blk + 4 * (a.off + (wq - a.wlo));
                row[0] |= (uint32_t)run;
                row[1] |= (uint32_t)(run >> 32);
                row[2] |= (uint32_t)(run >> 64);
                row[3] |= (uint32_t)(run >> 96);
            }
        }
    }
}

// Kept-pair scan of one (query tile, key tile) pair from its row segments: whether any pair is
// kept, whether the tile is complete and wholly kept, and the number of kept pairs. Key segments
// at a frame offset (key frame - query frame) listed in skip_dt count as not kept.
void scan_tile(const vdit_plan& p, const std::vector<Seg>& qs, const std::vector<Seg>& ks, bool complete,
               const std::vector<int>* skip_dt, bool& any, bool& all, long long& kept) {
    const bool causal = p.m.kind & VDIT_MASK_BLOCK_CAUSAL;
    any = false;
    all = complete;
    kept = 0;
    for (const Seg& a : qs) {
        for (const Seg& b : ks) {
            if (b.t < 0) { all = false; continue; }
            if (skip_dt && std::find(skip_dt->begin(), skip_dt->end(), b.t - a.t) != skip_dt->end()) {
                all = false;
                continue;
            }
            if (causal && b.t / p.m.chunk_frames > a.t / p.m.chunk_frames) {
                all = false;
                continue;
            }
            const int r = p.radius[std::abs(a.t - b.t)];
            if (std::abs(a.h - b.h) > r) { all = false; continue; }
            const int dmin = std::max(0, std::max(b.wlo - a.whi, a.wlo - b.whi));
            const int dmax = std::max(a.whi - b.wlo, b.whi - a.wlo);
            if (dmin <= r) {
                any = true;
                kept += pairs_within(a.wlo, a.whi, b.wlo, b.whi, r);
            }
            if (dmax > r) all = false;
        }
    }
}

// Hash of one 512-word keep-mask block: FNV-1a-style over 64-bit words in four interleaved lanes
// (independent multiply chains), folded into one value. Equal blocks are confirmed word by word.
uint64_t block_hash(const uint32_t* blk) {
    uint64_t lane[4] = {1469598103934665603ull, 1469598103934665603ull ^ 1, 1469598103934665603ull ^ 2,
                        1469598103934665603ull ^ 3};
    for (int wi = 0; wi < 512; wi += 8)
        for (int l = 0; l < 4; ++l)
            lane[l] = (lane[l] ^ ((uint64_t)blk[wi + 2 * l] | (uint64_t)blk[wi + 2 * l + 1] << 32)) *
                      1099511628211ull;
    return ((lane[0] * 31 + lane[1]) * 31 + lane[2]) * 31 + lane[3];
}

// Stores block `blk` (hash h) in `pool` once: returns the number of an identical block already in
// the pool, else appends it and returns its new number.
int dedupe_block(std::vector<uint32_t>& pool, std::unordered_map<uint64_t, std::vector<int>>& seen,
                 const uint32_t* blk, uint64_t h) {
    auto& same = seen[h];
    for (int b : same)
        if (std::equal(blk, blk + 512, pool.begin() + (size_t)b * 512)) return b;
    const int block = (int)(pool.size() / 512);
    pool.insert(pool.end(), blk, blk + 512);
    same.push_back(block);
    return block;
}

// What one query tile contributes to the plan, computed independently of the other tiles (so the
// tiles are computed in parallel) and merged into the plan in tile order (so the result, block
// numbering included, does not depend on the threads).
struct QtOut {
    // schedule of the mask as it is: listed key tiles, full flags, kept pairs; the keep-mask
    // blocks of the partial ones (512 words each, in list order) and their hashes
    std::vector<int> kt;
    std::vector<unsigned char> full;
    long long kept = 0;
    std::vector<uint32_t> blocks;
    std::vector<uint64_t> hashes;
    // kernel work list when single-patch entries pay off (dts not empty): aligned entries (key
    // row, partial or not) without the single-patch pairs, then one entry per offset in dts with
    // first key row diag_key; wblocks / whashes: the partial aligned entries' blocks, then one
    // block per offset
    std::vector<int> dts, wkey, diag_key;
    std::vector<unsigned char> wpartial;
    std::vector<uint32_t> wblocks;
    std::vector<uint64_t> whashes;
};

void plan_qtile(const vdit_plan& p, int qt, const std::vector<std::vector<Seg>>& kseg, bool single_patch,
                std::vector<Seg>& qs, QtOut& o) {
    const vdit_mask* m = &p.m;
    const int ft = p.g.grid_h * p.g.grid_w;
    const bool causal = m->kind & VDIT_MASK_BLOCK_CAUSAL;
    const int q0 = qt * VDIT_TILE, q1 = std::min(p.q_tokens, q0 + VDIT_TILE);
    segments(q0, q1, p.g.grid_h, p.g.grid_w, [&](int f) { return p.q_start + f; }, qs);
    o = QtOut();
    for (int kt = 0; kt < p.n_kt; ++kt) {
        const int k0 = kt * VDIT_TILE, k1 = std::min(p.kv_tokens, k0 + VDIT_TILE);
        bool any, all;
        long long kept;
        scan_tile(p, qs, kseg[kt], (q1 - q0 == VDIT_TILE) && (k1 - k0 == VDIT_TILE), nullptr, any, all, kept);
        o.kept += kept;
        if (!any) continue;
        o.kt.push_back(kt);
        o.full.push_back(all ? 1 : 0);
        if (!all) {
            // keep-mask block of this tile; identical blocks (tiles at the same offsets within
            // their frames with the same radii) are stored once at the merge, so the blocks the
            // kernel reads for all heads stay resident in L2
            tile_mask(p, qs, kseg[kt], o.blocks);
            o.hashes.push_back(block_hash(o.blocks.data() + o.blocks.size() - 512));
        }
    }
    const int n_export = (int)o.kt.size();
    // frame offsets dt (key frame - query frame) whose radial window is one patch: the kept
    // pairs at dt are (q, q + dt frames), one contiguous run of 128 key rows when the key
    // frames of the tile's (at most two) query frames sit in consecutive ring slots
    const int fa = q0 / ft, fb = (q1 - 1) / ft;
    const int ta = p.q_start + fa, tb = p.q_start + fb;
    if (single_patch) {
        for (int dt = p.kv_first - tb; dt <= p.kv_last - ta; ++dt) {
            if (p.radius[std::abs(dt)] != 0 || ta + dt < 0) continue;
            const int sa = (ta + dt) % p.cap_frames;
            if (fb != fa && sa == p.cap_frames - 1) continue;  // the run wraps the ring
            bool valid = false;
            for (int t = ta; t <= tb && !valid; ++t) {
                const int kf = t + dt;
                valid = kf >= p.kv_first && kf <= p.kv_last &&
                        !(causal && kf / m->chunk_frames > t / m->chunk_frames);
            }
            if (valid) o.dts.push_back(dt);
        }
    }
    // kernel work list: the aligned tiles without the single-patch pairs, plus one entry per
    // offset, kept only when it shortens the list
    if (o.dts.empty()) return;
    for (int kt = 0; kt < p.n_kt; ++kt) {
        const int k0 = kt * VDIT_TILE, k1 = std::min(p.kv_tokens, k0 + VDIT_TILE);
        bool any, all;
        long long kept;
        scan_tile(p, qs, kseg[kt], (q1 - q0 == VDIT_TILE) && (k1 - k0 == VDIT_TILE), &o.dts, any, all, kept);
        if (!any) continue;
        o.wkey.push_back(k0);
        o.wpartial.push_back(all ? 0 : 1);
        if (!all) {
            tile_mask(p, qs, kseg[kt], o.wblocks, &o.dts);
            o.whashes.push_back(block_hash(o.wblocks.data() + o.wblocks.size() - 512));
        }
    }
    if ((int)(o.wkey.size() + o.dts.size()) >= n_export) {  // no gain: plain tiles
        o.dts.clear();
        o.wkey.clear();
        o.wpartial.clear();
        o.wblocks.clear();
        o.whashes.clear();
        return;
    }
    for (int dt : o.dts) {
        // row r (query q0 + r at frame t) keeps key row k_start + r, its own patch at frame
        // t + dt, if that frame is held and the chunk order allows it
        const int k_start = ((ta + dt) % p.cap_frames) * ft + (q0 - fa * ft);
        const size_t at = o.wblocks.size();
        o.wblocks.resize(at + 512, 0u);
        for (int r = 0; r < q1 - q0; ++r) {
            const int t = p.q_start + (q0 + r) / ft, kf = t + dt;
            const bool keep = kf >= p.kv_first && kf <= p.kv_last &&
                              !(causal && kf / m->chunk_frames > t / m->chunk_frames) &&
                              k_start + r < p.kv_tokens;
            if (keep) o.wblocks[at + 4 * r + (r >> 5)] |= 1u << (r & 31);
        }
        o.diag_key.push_back(k_start);
        o.whashes.push_back(block_hash(o.wblocks.data() + at));
    }
}

}  // namespace

extern "C" int vdit_attn_plan(vdit_plan** out, const vdit_geom* g, const vdit_mask* m,
                              int q_start_frame, int q_frames, int capacity_frames,
                              int kv_first_frame, int kv_last_frame) {
    using vdit::fail;
    if (!out) return fail(VDIT_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    if (int rc = vdit::check_geom(g)) return rc;
    if (!m) return fail(VDIT_ERR_INVALID_ARG, "mask is NULL");
    if (m->kind & ~(VDIT_MASK_BLOCK_CAUSAL | VDIT_MASK_RADIAL | VDIT_MASK_DYNAMIC))
        return fail(VDIT_ERR_INVALID_ARG, "unknown mask kind bits");
    if ((m->kind & VDIT_MASK_DYNAMIC) && !(m->tau > 0.0 && m->tau < 1e30))
        return fail(VDIT_ERR_INVALID_ARG, "dynamic threshold needs a finite tau > 0");
    if ((m->kind & VDIT_MASK_BLOCK_CAUSAL) && m->chunk_frames < 1)
        return fail(VDIT_ERR_INVALID_ARG, "chunk_frames must be >= 1");
    if ((m->kind & VDIT_MASK_RADIAL) && (m->w0 < 0 || m->gamma_shift < 0 || m->lambda < 0))
        return fail(VDIT_ERR_INVALID_ARG, "radial mask needs w0, gamma_shift, lambda >= 0");
    if (q_start_frame < 0 || q_frames < 1 || q_start_frame + q_frames - 1 > VDIT_MAX_FRAME)
        return fail(VDIT_ERR_INVALID_ARG, "query frames out of range");
    if (capacity_frames < 1 || kv_first_frame < 0 || kv_last_frame < kv_first_frame ||
        kv_last_frame - kv_first_frame + 1 > capacity_frames || kv_last_frame > VDIT_MAX_FRAME)
        return fail(VDIT_ERR_INVALID_ARG, "KV window must satisfy 0 <= first <= last, "
                                          "last - first < capacity_frames");

    vdit_plan* p = new (std::nothrow) vdit_plan();
    if (!p) return fail(VDIT_ERR_INVALID_ARG, "out of host memory");
    // host allocations below may fail (bad_alloc); the C ABI reports that instead of throwing
    try {
        p->g = *g;
        p->m = *m;
        p->q_start = q_start_frame;
        p->q_frames = q_frames;
        p->cap_frames = capacity_frames;
        p->kv_first = kv_first_frame;
        p->kv_last = kv_last_frame;
        const int ft = g->grid_h * g->grid_w;
        const long long qtok = (long long)q_frames * ft, ktok = (long long)capacity_frames * ft;
        if (qtok > INT_MAX / 2 || ktok > INT_MAX / 2) {
            delete p;
            return fail(VDIT_ERR_UNSUPPORTED, "too many tokens");
        }
        p->q_tokens = (int)qtok;
        p->kv_tokens = (int)ktok;
        p->n_qt = (p->q_tokens + VDIT_TILE - 1) / VDIT_TILE;
        p->n_kt = (p->kv_tokens + VDIT_TILE - 1) / VDIT_TILE;

        p->slot_frame.assign(capacity_frames, -1);
        for (int f = kv_first_frame; f <= kv_last_frame; ++f) p->slot_frame[f % capacity_frames] = f;

        const int q_last = q_start_frame + q_frames - 1;
        p->dt_max = std::max(std::abs(q_last - kv_first_frame), std::abs(kv_last_frame - q_start_frame));
        if (p->dt_max > VDIT_MAX_DT) {
            delete p;
            return fail(VDIT_ERR_UNSUPPORTED, "query and key frames further apart than VDIT_MAX_DT");
        }
        p->radius.resize(p->dt_max + 1);
        for (int dt = 0; dt <= p->dt_max; ++dt) p->radius[dt] = radius_at(*m, dt);

        std::vector<std::vector<Seg>> kseg(p->n_kt);
        for (int kt = 0; kt < p->n_kt; ++kt)
            segments(kt * VDIT_TILE, std::min(p->kv_tokens, (kt + 1) * VDIT_TILE), g->grid_h,
                     g->grid_w, [&](int slot) { return p->slot_frame[slot]; }, kseg[kt]);
        std::unordered_map<uint64_t, std::vector<int>> seen, kseen;  // mask block hash -> block numbers
        p->row_ptr.assign(p->n_qt + 1, 0);
        p->w_row_ptr.assign(p->n_qt + 1, 0);
        p->w_aligned.assign(p->n_qt, 0);
        p->kept_pairs = 0;
        p->n_full = 0;
        // single-patch entries need a q-tile to span at most two frames (128 <= tokens per frame)
        const bool single_patch = (m->kind & VDIT_MASK_RADIAL) && ft >= VDIT_TILE;
        // q-tiles are computed in batches by a few host threads, then merged in order
        int n_threads = (int)std::max(1u, std::min(16u, std::thread::hardware_concurrency()));
        if (const char* env = std::getenv("VDIT_PLAN_THREADS")) {
            const int want = std::atoi(env);
            if (want >= 1) n_threads = std::min(want, 64);
        }
        const int batch = std::max(1, std::min(p->n_qt, 8 * n_threads));
        std::vector<QtOut> outs(batch);
        std::vector<std::vector<Seg>> qsegs(n_threads);
        for (int b0 = 0; b0 < p->n_qt; b0 += batch) {
            const int nb = std::min(batch, p->n_qt - b0);
            std::atomic<int> next{0};
            std::atomic<bool> failed{false};
            auto work = [&](int tid) {
                try {
                    for (int i = next++; i < nb; i = next++) plan_qtile(*p, b0 + i, kseg, single_patch, qsegs[tid], outs[i]);
                } catch (...) {
                    failed = true;
                }
            };
            const int nt = std::min(n_threads, nb);
            std::vector<std::thread> pool;
            try {
                for (int t = 1; t < nt; ++t) pool.emplace_back(work, t);
            } catch (...) {
                failed = true;  // no further thread: the calling thread does the rest
            }
            work(0);
            for (auto& th : pool) th.join();
            if (failed) throw std::bad_alloc();
            // merge in q-tile order
            for (int i = 0; i < nb; ++i) {
                const int qt = b0 + i;
                const QtOut& o = outs[i];
                p->kept_pairs += o.kept;
                const size_t first = p->col_idx.size();
                for (size_t e = 0, pb = 0; e < o.kt.size(); ++e) {
                    p->col_idx.push_back(o.kt[e]);
                    p->full.push_back(o.full[e]);
                    p->n_full += o.full[e];
                    int block = -1;
                    if (!o.full[e]) {
                        block = dedupe_block(p->masks, seen, o.blocks.data() + 512 * pb, o.hashes[pb]);
                        ++pb;
                    }
                    p->mask_of.push_back(block);
                }
                p->row_ptr[qt + 1] = (int)p->col_idx.size();
                if (o.dts.empty()) {
                    p->w_aligned[qt] = (int)o.kt.size();
                    for (size_t e = first, pb = 0; e < p->col_idx.size(); ++e) {
                        p->w_key.push_back(p->col_idx[e] * VDIT_TILE);
                        int block = -1;
                        if (!p->full[e]) {
                            block = dedupe_block(p->kmasks, kseen, o.blocks.data() + 512 * pb, o.hashes[pb]);
                            ++pb;
                        }
                        p->w_mask.push_back(block);
                    }
                } else {
                    p->w_aligned[qt] = (int)o.wkey.size();
                    size_t pb = 0;
                    for (size_t e = 0; e < o.wkey.size(); ++e) {
                        p->w_key.push_back(o.wkey[e]);
                        int block = -1;
                        if (o.wpartial[e]) {
                            block = dedupe_block(p->kmasks, kseen, o.wblocks.data() + 512 * pb, o.whashes[pb]);
                            ++pb;
                        }
                        p->w_mask.push_back(block);
                    }
                    for (size_t d = 0; d < o.dts.size(); ++d, ++pb) {
                        p->w_key.push_back(o.diag_key[d]);
                        p->w_mask.push_back(dedupe_block(p->kmasks, kseen, o.wblocks.data() + 512 * pb, o.whashes[pb]));
                        ++p->n_diag;
                    }
                }
                p->w_row_ptr[qt + 1] = (int)p->w_key.size();
            }
        }
        // union lists of q-tile pairs, from the kernel's work list: entries at the same (aligned) key
        // row merge; an unaligned single-patch entry stays on its own (one q-tile)
        p->n_qb = (p->n_qt + 1) / 2;
        p->u_row_ptr.assign(p->n_qb + 1, 0);
        for (int b = 0; b < p->n_qb; ++b) {
            const int t0 = 2 * b, t1 = 2 * b + 1;
            // aligned entries of the two q-tiles, merged by key row (both ascending)
            int i = p->w_row_ptr[t0], ie = i + p->w_aligned[t0];
            int k = t1 < p->n_qt ? p->w_row_ptr[t1] : 0, ke = t1 < p->n_qt ? k + p->w_aligned[t1] : 0;
            while (i < ie || k < ke) {
                const int ci = i < ie ? p->w_key[i] : INT_MAX, ck = k < ke ? p->w_key[k] : INT_MAX;
                const int c = std::min(ci, ck);
                unsigned char f = 0;
                int m0 = -1, m1 = -1;
                if (ci == c) { f |= 1 | (p->w_mask[i] < 0 ? 2 : 0); m0 = p->w_mask[i]; ++i; }
                if (ck == c) { f |= 4 | (p->w_mask[k] < 0 ? 8 : 0); m1 = p->w_mask[k]; ++k; }
                p->u_col.push_back(c);
                p->u_flags.push_back(f);
                p->u_mask.push_back(m0);
                p->u_mask.push_back(m1);
            }
            // single-patch entries, each for one q-tile
            for (int x = 0; x < 2; ++x) {
                const int qt = t0 + x;
                if (qt >= p->n_qt) break;
                for (int e = p->w_row_ptr[qt] + p->w_aligned[qt]; e < p->w_row_ptr[qt + 1]; ++e) {
                    p->u_col.push_back(p->w_key[e]);
                    p->u_flags.push_back((unsigned char)(x ? 4 : 1));
                    p->u_mask.push_back(x ? -1 : p->w_mask[e]);
                    p->u_mask.push_back(x ? p->w_mask[e] : -1);
                }
            }
            p->u_row_ptr[b + 1] = (int)p->u_col.size();
        }
        p->unit_order.resize(p->n_qb);
        for (int i = 0; i < p->n_qb; ++i) p->unit_order[i] = i;
        std::stable_sort(p->unit_order.begin(), p->unit_order.end(), [&](int a, int b) {
            return p->u_row_ptr[a + 1] - p->u_row_ptr[a] > p->u_row_ptr[b + 1] - p->u_row_ptr[b];
        });
        *out = p;
        return VDIT_OK;
    } catch (const std::bad_alloc&) {
        delete p;
        return fail(VDIT_ERR_UNSUPPORTED, "out of host memory while building the plan");
    }
}

namespace {

// CTA schedule of the attention kernel on a device with `sms` SMs, one CTA per SM at a time.
// A unit is one q-block (two 128-query tiles) of one head with its union list of n entries; the
// CTAs go out in launch order, each to the SM that frees first, so the kernel's time is the
// makespan of that list schedule. A CTA costs its entries plus kPieceTiles (prologue: Q load and
// RoPE, TMEM allocation, pipeline fill; epilogue: O write). Units go in head-major order (the
// CTAs in flight then share few heads' K / V in L2), longest list first within a head.
//
// Whole units alone leave the SMs idle at the end (1 536 equal units over 148 SMs: 10.4 waves,
// the last 38% full). So the schedule picks a level T and walks the units in order: a unit that
// ends by T on the first free SM runs whole; one that does not is cut into pieces (each at least
// kMinPiece entries), each piece filling the SM that frees next up to T. A piece writes its
// normalised partial O and log2-sum-exp in fp32 into a slot of the workspace, and a second
// kernel merges the pieces of every cut unit. The level is the smallest T (binary search) at
// which every unit fits within kMaxSlots partial slots; the split schedule is kept when its
// estimated time (makespan plus the partial results written and read back, plus one launch) is
// below the whole-unit schedule's. The dynamic-threshold mode never cuts: its threshold needs
// each row's maximum over all its candidates. Constants measured on a B200 (one CTA runs a union
// entry of two 128-query tiles in ~1.44 us, ~12 entries' worth of fixed cost per CTA).
struct Schedule {
    std::vector<int> cta;    // per CTA: q-block, head, first entry (within the unit), entries, slot
    std::vector<int> merge;  // per cut unit: q-block, head, first slot, pieces
    int slots = 0, max_pieces = 1;
    double span = 0.0;       // makespan, in entry times
};

constexpr double kPieceTiles = 12.0, kTileSeconds = 1.44e-6, kBytesPerSecond = 6.5e12,
                 kLaunchSeconds = 4e-6;
constexpr int kMinPiece = 8;

// List schedule at level T (T <= 0: whole units only). false if some unit cannot be placed by
// the rule (a cut unit needs more than max_slots slots, or the first free SM has no room left
// for a piece).
bool schedule_at(const vdit_plan& p, int sms, double T, int max_slots, Schedule* out) {
    std::vector<double> f(std::max(1, sms), 0.0);  // min-heap of the SMs' free times
    auto less = std::greater<double>();
    Schedule s;
    s.cta.reserve(5 * (size_t)p.n_qb * p.g.heads);
    for (int h = 0; h < p.g.heads; ++h)
        for (int i = 0; i < p.n_qb; ++i) {
            const int u = p.unit_order[i];
            const int n = p.u_row_ptr[u + 1] - p.u_row_ptr[u];
            std::pop_heap(f.begin(), f.end(), less);
            double& t = f.back();
            // whole: when it ends by T, or is too short to cut (an empty list included; its CTA
            // still writes o = 0 and lse = -inf)
            if (T <= 0.0 || t + n + kPieceTiles <= T || n < 2 * kMinPiece) {
                t += n + kPieceTiles;
                s.span = std::max(s.span, t);
                std::push_heap(f.begin(), f.end(), less);
                s.cta.insert(s.cta.end(), {u, h, 0, n, -1});
                continue;
            }
            std::push_heap(f.begin(), f.end(), less);
            const int first_slot = s.slots;
            int done = 0, pieces = 0;
            while (done < n) {
                std::pop_heap(f.begin(), f.end(), less);
                double& tf = f.back();
                const int rem = n - done;
                const double room = T - tf - kPieceTiles;
                int take;
                if (room >= rem) take = rem;                                   // the rest fits
                else if (room >= kMinPiece && rem >= 2 * kMinPiece)
                    take = std::min((int)room, rem - kMinPiece);               // leave >= kMinPiece
                else return false;
                if (s.slots >= max_slots) return false;
                tf += take + kPieceTiles;
                s.span = std::max(s.span, tf);
                std::push_heap(f.begin(), f.end(), less);
                s.cta.insert(s.cta.end(), {u, h, done, take, s.slots++});
                done += take;
                ++pieces;
            }
            if (pieces == 1) {  // the whole unit fitted after all: no partial result needed
                --s.slots;
                s.cta.back() = -1;
            } else {
                s.merge.insert(s.merge.end(), {u, h, first_slot, pieces});
                s.max_pieces = std::max(s.max_pieces, pieces);
            }
        }
    *out = std::move(s);
    return true;
}

double schedule_seconds(const vdit_plan& p, const Schedule& s) {
    double t = s.span * kTileSeconds;
    if (s.slots > 0)
        t += 2.0 * s.slots * 256.0 * (p.g.head_dim + 1) * 4.0 / kBytesPerSecond + kLaunchSeconds;
    return t;
}

Schedule build_schedule(const vdit_plan& p, int sms) {
    Schedule whole;
    schedule_at(p, sms, 0.0, 0, &whole);
    if (p.m.kind & VDIT_MASK_DYNAMIC) return whole;
    double work = 0.0;
    for (int b = 0; b < p.n_qb; ++b) work += p.u_row_ptr[b + 1] - p.u_row_ptr[b] + kPieceTiles;
    double lo = work * p.g.heads / std::max(1, sms), hi = whole.span;
    const int max_slots = vdit::max_partial_slots(p.g.head_dim);
    Schedule best = whole, s;
    double best_t = schedule_seconds(p, whole);
    for (int it = 0; it < 40 && hi - lo > 0.5; ++it) {
        const double mid = 0.5 * (lo + hi);
        if (schedule_at(p, sms, mid, max_slots, &s)) {
            hi = mid;
            const double t = schedule_seconds(p, s);
            if (t < best_t) { best_t = t; best = std::move(s); }
        } else {
            lo = mid;
        }
    }
    return best;
}

void apply_schedule(vdit_plan* p, Schedule&& s) {
    p->cta = std::move(s.cta);
    p->merge = std::move(s.merge);
    p->n_slots = s.slots;
    p->n_split = s.max_pieces;
}

}  // namespace

extern "C" int vdit_plan_export_schedule(const vdit_plan* p, int sm_count, int* n_ctas, int* n_cut_units,
                                         int* cta, int* merge) {
    if (!p || !n_ctas || !n_cut_units || sm_count < 1)
        return vdit::fail(VDIT_ERR_INVALID_ARG, "NULL plan or count, or sm_count < 1");
    const Schedule s = build_schedule(*p, sm_count);
    *n_ctas = (int)(s.cta.size() / 5);
    *n_cut_units = (int)(s.merge.size() / 4);
    if (cta) std::memcpy(cta, s.cta.data(), sizeof(int) * s.cta.size());
    if (merge && !s.merge.empty()) std::memcpy(merge, s.merge.data(), sizeof(int) * s.merge.size());
    return VDIT_OK;
}

extern "C" int vdit_plan_info(const vdit_plan* p, vdit_plan_info_t* info) {
    if (!p || !info) return vdit::fail(VDIT_ERR_INVALID_ARG, "NULL plan or info");
    info->q_tokens = p->q_tokens;
    info->kv_tokens = p->kv_tokens;
    info->q_tiles = p->n_qt;
    info->kv_tiles = p->n_kt;
    info->tiles = (int)p->col_idx.size();
    info->full_tiles = p->n_full;
    info->kept_pairs = p->kept_pairs;
    info->uploaded = p->d_buf != nullptr;
    info->kv_splits = p->n_split;
    info->workspace_bytes = (long long)p->ws_bytes;
    info->ctas = (int)(p->cta.size() / 5);
    info->cut_units = (int)(p->merge.size() / 4);
    info->mask_bytes = (long long)(sizeof(uint32_t) * p->masks.size());
    info->work_entries = (int)p->w_key.size();
    info->single_patch_entries = p->n_diag;
    info->work_mask_bytes = (long long)(sizeof(uint32_t) * p->kmasks.size());
    return VDIT_OK;
}

extern "C" int vdit_plan_export_work(const vdit_plan* p, int* row_ptr, int* key_row, int* mask_index,
                                     unsigned int* words) {
    if (!p || !row_ptr || (!p->w_key.empty() && (!key_row || !mask_index)) || (!p->kmasks.empty() && !words))
        return vdit::fail(VDIT_ERR_INVALID_ARG, "NULL plan or output");
    std::memcpy(row_ptr, p->w_row_ptr.data(), sizeof(int) * p->w_row_ptr.size());
    if (!p->w_key.empty()) {
        std::memcpy(key_row, p->w_key.data(), sizeof(int) * p->w_key.size());
        std::memcpy(mask_index, p->w_mask.data(), sizeof(int) * p->w_mask.size());
    }
    if (!p->kmasks.empty()) std::memcpy(words, p->kmasks.data(), sizeof(uint32_t) * p->kmasks.size());
    return VDIT_OK;
}

extern "C" int vdit_plan_export_masks(const vdit_plan* p, int* mask_index, unsigned int* words) {
    if (!p || (!p->mask_of.empty() && !mask_index) || (!p->masks.empty() && !words))
        return vdit::fail(VDIT_ERR_INVALID_ARG, "NULL plan or output");
    if (!p->mask_of.empty()) std::memcpy(mask_index, p->mask_of.data(), sizeof(int) * p->mask_of.size());
    if (!p->masks.empty()) std::memcpy(words, p->masks.data(), sizeof(uint32_t) * p->masks.size());
    return VDIT_OK;
}

extern "C" int vdit_plan_export(const vdit_plan* p, int* row_ptr, int* col_idx,
                                unsigned char* full) {
    if (!p || !row_ptr || (!p->col_idx.empty() && (!col_idx || !full)))
        return vdit::fail(VDIT_ERR_INVALID_ARG, "NULL plan or output");
    std::memcpy(row_ptr, p->row_ptr.data(), sizeof(int) * p->row_ptr.size());
    if (!p->col_idx.empty()) {
        std::memcpy(col_idx, p->col_idx.data(), sizeof(int) * p->col_idx.size());
        std::memcpy(full, p->full.data(), p->full.size());
    }
    return VDIT_OK;
}

extern "C" int vdit_plan_upload(vdit_plan* p, void* stream) {
    using vdit::cuda_check;
    if (!p) return vdit::fail(VDIT_ERR_INVALID_ARG, "NULL plan");
    int dev = 0;
    if (int rc = cuda_check(cudaGetDevice(&dev), "cudaGetDevice")) return rc;
    if (p->d_buf) {
        if (p->device == dev) return VDIT_OK;
        return vdit::fail(VDIT_ERR_INVALID_ARG, "plan already uploaded to another device");
    }
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // the attention kernels' per-device set-up happens here, in a call that allocates anyway, so
    // that the forward calls on this plan (the no-allocation one included) only launch
    if (int rc = vdit::attn_prepare_device(dev)) return rc;
    apply_schedule(p, build_schedule(*p, sms));
    // one allocation of what the kernels read: u_row_ptr | u_col | u_flags | CTA table (int4) |
    // CTA slots | merge table (int4) | u_mask | masks | (workspace: partial O | partial lse); the
    // per-q-tile lists, the slot frames and the radius table stay on the host (exports, mask
    // construction)
    auto up = [](size_t n) { return (n + 255) / 256 * 256; };
    const int n_cta = (int)(p->cta.size() / 5), n_cut = (int)(p->merge.size() / 4);
    std::vector<int> cta4(4 * (size_t)n_cta), slot(n_cta);
    for (int c = 0; c < n_cta; ++c) {
        for (int k = 0; k < 4; ++k) cta4[4 * (size_t)c + k] = p->cta[5 * (size_t)c + k];
        slot[c] = p->cta[5 * (size_t)c + 4];
    }
    const size_t n_urp = sizeof(int) * p->u_row_ptr.size();
    const size_t n_uc = sizeof(int) * std::max<size_t>(1, p->u_col.size());
    const size_t n_uf = std::max<size_t>(1, p->u_flags.size());
    const size_t n_ct = sizeof(int) * std::max<size_t>(4, cta4.size());
    const size_t n_cs = sizeof(int) * std::max<size_t>(1, slot.size());
    const size_t n_mg = sizeof(int) * std::max<size_t>(4, p->merge.size());
    const size_t n_um = sizeof(int) * std::max<size_t>(1, p->u_mask.size());
    const size_t n_mk = sizeof(uint32_t) * std::max<size_t>(4, p->kmasks.size());
    const size_t n_wo = sizeof(float) * (size_t)p->n_slots * 256 * p->g.head_dim;
    const size_t n_wl = sizeof(float) * (size_t)p->n_slots * 256;
    const size_t meta = up(n_urp) + up(n_uc) + up(n_uf) + up(n_ct) + up(n_cs) + up(n_mg) + up(n_um) + up(n_mk);
    const size_t total = meta + up(n_wo) + up(n_wl);
    std::vector<unsigned char> host(meta, 0);
    size_t off = 0;
    auto put = [&](const void* src, size_t n, size_t reserved) {
        size_t at = off;
        if (n) std::memcpy(host.data() + off, src, n);
        off += up(reserved);
        return at;
    };
    const size_t o_urp = put(p->u_row_ptr.data(), n_urp, n_urp);
    const size_t o_uc = put(p->u_col.data(), sizeof(int) * p->u_col.size(), n_uc);
    const size_t o_uf = put(p->u_flags.data(), p->u_flags.size(), n_uf);
    const size_t o_ct = put(cta4.data(), sizeof(int) * cta4.size(), n_ct);
    const size_t o_cs = put(slot.data(), sizeof(int) * slot.size(), n_cs);
    const size_t o_mg = put(p->merge.data(), sizeof(int) * p->merge.size(), n_mg);
    const size_t o_um = put(p->u_mask.data(), sizeof(int) * p->u_mask.size(), n_um);
    const size_t o_mk = put(p->kmasks.data(), sizeof(uint32_t) * p->kmasks.size(), n_mk);
    if (off != meta) return vdit::fail(VDIT_ERR_INVALID_ARG, "internal: plan layout mismatch");
    // the workspace is not initialised: a piece writes every partial row it owns before the merge
    void* d = nullptr;
    if (int rc = cuda_check(cudaMalloc(&d, total), "cudaMalloc(plan)")) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (int rc = cuda_check(cudaMemcpyAsync(d, host.data(), meta, cudaMemcpyHostToDevice, s),
                            "cudaMemcpyAsync(plan)")) {
        cudaFree(d);
        return rc;
    }
    // a pageable source is staged before cudaMemcpyAsync returns, so `host` may go now
    unsigned char* b = static_cast<unsigned char*>(d);
    p->device = dev;
    p->d_buf = d;
    p->d_u_row_ptr = reinterpret_cast<const int*>(b + o_urp);
    p->d_u_col = reinterpret_cast<const int*>(b + o_uc);
    p->d_u_flags = b + o_uf;
    p->d_cta = reinterpret_cast<const int*>(b + o_ct);
    p->d_cta_slot = reinterpret_cast<const int*>(b + o_cs);
    p->d_merge = reinterpret_cast<const int*>(b + o_mg);
    p->d_u_mask = reinterpret_cast<const int*>(b + o_um);
    p->d_masks = reinterpret_cast<const uint32_t*>(b + o_mk);
    p->ws_bytes = p->n_slots ? up(n_wo) + n_wl : 0;
    if (p->n_slots) {
        p->d_ws_o = reinterpret_cast<float*>(b + meta);
        p->d_ws_lse = reinterpret_cast<float*>(b + meta + up(n_wo));
    }
    return VDIT_OK;
}

extern "C" void vdit_plan_destroy(vdit_plan* p) {
    if (!p) return;
    if (p->d_buf) {
        int cur = 0;
        cudaGetDevice(&cur);
        cudaSetDevice(p->device);
        cudaFree(p->d_buf);
        cudaSetDevice(cur);
    }
    delete p;
}
