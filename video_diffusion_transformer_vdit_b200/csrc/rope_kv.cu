// 3-D RoPE with a global time index and the KV-cache append (libvdit, sm_100a).
//
// "Accelerating Video Generation Inference with Sequential-Parallel 3D Positional Encoding Using
// a Global Time Index": section 2.B gives each chunk its own temporal positions from its start
// frame (t = s + local frame) so no gather of the sequence is needed before RoPE; section 2.C
// precomputes the rotary frequencies into contiguous tables; section 2.A keeps a KV cache of
// past chunks. "Timeripple" (Metodologia 1) splits the channels into a temporal group and two
// spatial groups.
//
// Both kernels are HBM streams: every 16-byte chunk of [tokens, heads, head_dim] is read once and
// written once, consecutive lanes on consecutive chunks, several independent loads in flight
// per lane (the kernels are latency-bound otherwise). Each 32-bit word of a chunk is one RoPE
// pair (channel 2j in the low half, 2j+1 in the high half), rotated in fp32 with a (cos, sin)
// pair read from the tables (L1/L2 resident) and rounded to bf16 nearest-even.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"

namespace vdit {

namespace {
std::mutex g_tab_mu;
std::map<std::tuple<int, int, int, int, uint64_t>, RopeTables> g_tabs;
}  // namespace

int get_rope_tables(const vdit_geom* g, RopeTables* out) {
    int dev = 0;
    if (int rc = cuda_check(cudaGetDevice(&dev), "cudaGetDevice")) return rc;
    uint64_t tbits;
    std::memcpy(&tbits, &g->theta, sizeof tbits);
    auto key = std::make_tuple(dev, g->band_t, g->band_h, g->band_w, tbits);
    std::lock_guard<std::mutex> lk(g_tab_mu);
    auto it = g_tabs.find(key);
    if (it != g_tabs.end()) {
        *out = it->second;
        return VDIT_OK;
    }
    const int bt2 = g->band_t / 2, bh2 = g->band_h / 2, bw2 = g->band_w / 2;
    const size_t nt = (size_t)(VDIT_MAX_FRAME + 1) * bt2, nh = (size_t)VDIT_MAX_GRID * bh2,
                 nw = (size_t)VDIT_MAX_GRID * bw2;
    std::vector<float2> host(nt + nh + nw);
    auto fill = [&](float2* dst, int rows, int width) {
        for (int p = 0; p < rows; ++p)
            for (int j = 0; j < width / 2; ++j) {
                const double omega = std::pow(g->theta, -2.0 * j / width);
                const double a = (double)p * omega;
                dst[(size_t)p * (width / 2) + j] = make_float2((float)std::cos(a), (float)std::sin(a));
            }
    };
    fill(host.data(), VDIT_MAX_FRAME + 1, g->band_t);
    fill(host.data() + nt, VDIT_MAX_GRID, g->band_h);
    fill(host.data() + nt + nh, VDIT_MAX_GRID, g->band_w);
    void* d = nullptr;
    if (int rc = cuda_check(cudaMalloc(&d, host.size() * sizeof(float2)), "cudaMalloc(rope tables)"))
        return rc;
    if (int rc = cuda_check(cudaMemcpy(d, host.data(), host.size() * sizeof(float2),
                                       cudaMemcpyHostToDevice), "cudaMemcpy(rope tables)")) {
        cudaFree(d);
        return rc;
    }
    RopeTables t;
    t.t = d;
    t.h = static_cast<float2*>(d) + nt;
    t.w = static_cast<float2*>(d) + nt + nh;
    g_tabs[key] = t;
    *out = t;
    return VDIT_OK;
}

// Looks the tables up without building them: for callers that must not allocate. Fails if no
// earlier call on this device built them for this band set.
int find_rope_tables(const vdit_geom* g, RopeTables* out) {
    int dev = 0;
    if (int rc = cuda_check(cudaGetDevice(&dev), "cudaGetDevice")) return rc;
    uint64_t tbits;
    std::memcpy(&tbits, &g->theta, sizeof tbits);
    auto key = std::make_tuple(dev, g->band_t, g->band_h, g->band_w, tbits);
    std::lock_guard<std::mutex> lk(g_tab_mu);
    auto it = g_tabs.find(key);
    if (it == g_tabs.end())
        return fail(VDIT_ERR_INVALID_ARG,
                    "RoPE tables for these bands do not exist on this device yet; an earlier "
                    "vdit_kv_append, vdit_rope3d_apply or vdit_attn_forward call builds them");
    *out = it->second;
    return VDIT_OK;
}

}  // namespace vdit

namespace {

// Division by a run-time invariant d (Granlund and Montgomery, "Division by invariant integers
// using multiplication", PLDI 1994): with s = ceil(log2 d) and m = floor(2^(32+s) / d) + 1 - 2^32,
// n / d = (mulhi(n, m) + n) >> s for every n < 2^31 (the sum cannot overflow 32 bits there).
// All chunk, token and frame indices handled here are < 2^31 (checked on the host).
struct FastDiv {
    uint32_t m;
    uint32_t s;
    uint32_t d;
};
FastDiv make_fastdiv(uint32_t d) {
    FastDiv f;
    f.d = d;
    if (d <= 1) {
        f.m = 0;
        f.s = 0;
        return f;
    }
    uint32_t s = 0;
    while ((1ull << s) < d) ++s;
    f.s = s;
    f.m = (uint32_t)(((1ull << (32 + s)) / d) + 1 - (1ull << 32));
    return f;
}
__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv& f) {
    return f.d == 1 ? n : (__umulhi(n, f.m) + n) >> f.s;
}

struct StreamArgs {
    const uint4* x;     // rope: input; append: K chunk
    uint4* y;           // rope: output; append: K cache
    const uint4* v;     // append: V chunk
    uint4* vc;          // append: V cache
    int n_tokens;
    int cpr_log2;       // log2(head_dim / 8): 16-byte chunks per head row
    int cpt;            // chunks per token = heads * head_dim / 8
    int grid_h, grid_w;
    int start_frame;
    int cap_frames;     // append: ring capacity in frames
    long long cap_tok;  // append: capacity_frames * grid_h * grid_w
    FastDiv by_ft, by_w, by_cap;
    const float2* tt;
    const float2* th;
    const float2* tw;
    int bt2, bh2, bw2;  // pairs per band
};

// (cos, sin) of the four RoPE pairs pp0 .. pp0+3 of one 16-byte chunk at position (t, h, w).
__device__ __forceinline__ void chunk_angles(float2 (&cs)[4], int pp0, int t, int h, int w,
                                             const StreamArgs& a) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int pp = pp0 + i;
        // band of this pair, chosen without branches: the lanes of a warp hold different
        // chunks of a head row and would otherwise split over the three table lookups
        const bool in_h = pp >= a.bt2, in_w = pp >= a.bt2 + a.bh2;
        const float2* tab = in_w ? a.tw : (in_h ? a.th : a.tt);
        const int row = in_w ? w : (in_h ? h : t);
        const int width = in_w ? a.bw2 : (in_h ? a.bh2 : a.bt2);
        const int jj = pp - (in_w ? a.bt2 + a.bh2 : (in_h ? a.bt2 : 0));
        cs[i] = __ldg(tab + (size_t)row * width + jj);
    }
}

// Rotates the four pairs of one chunk: (x0, x1) -> (x0 cos - x1 sin, x0 sin + x1 cos) in fp32.
__device__ __forceinline__ uint4 rotate_chunk(uint4 in, const float2 (&cs)[4]) {
    uint32_t word[4] = {in.x, in.y, in.z, in.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 b;
        memcpy(&b, &word[i], 4);
        const float2 xv = __bfloat1622float2(b);
        const float y0 = fmaf(xv.x, cs[i].x, -xv.y * cs[i].y);
        const float y1 = fmaf(xv.x, cs[i].y, xv.y * cs[i].x);
        b = __floats2bfloat162_rn(y0, y1);
        memcpy(&word[i], &b, 4);
    }
    return make_uint4(word[0], word[1], word[2], word[3]);
}

// One warp streams one token's row of heads * head_dim / 8 chunks at a time: load u of lane l
// takes chunk 32u + l, so every warp access is 512 contiguous bytes, and since 32 is a multiple
// of the chunks per head row, a lane meets the same RoPE pairs in every head: its four (cos, sin)
// pairs and the token's (t, h, w) decode are done once per token, not once per chunk.
// kBatch independent 16-byte loads per lane and tensor are in flight before any store; the
// append holds two tensors' loads, so it runs half as many blocks per SM at twice the registers.
constexpr int kBatch = 8;
constexpr int kWarpsPerBlock = 8;
template <bool APPEND>
constexpr int blocks_per_sm() { return APPEND ? 2 : 4; }

// APPEND = false: y = RoPE(x) at t = start_frame + local frame.
// APPEND = true:  K' = RoPE(k) (ROTATE) or K' = k (already rotated, !ROTATE) and V (unchanged) go
//                 to frame slot t mod capacity of the caches.
template <bool APPEND, bool ROTATE = true>
__global__ void __launch_bounds__(kWarpsPerBlock * 32, blocks_per_sm<APPEND>())
    rope_stream_kernel(StreamArgs a) {
    const int lane = threadIdx.x & 31;
    const int n_warps = gridDim.x * kWarpsPerBlock;
    const int c8 = lane & ((1 << a.cpr_log2) - 1);
    const int ft = a.grid_h * a.grid_w;
    for (int tok = blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5); tok < a.n_tokens; tok += n_warps) {
        const uint32_t f = fdiv((uint32_t)tok, a.by_ft);
        const int rem = tok - (int)f * ft;
        const int h = (int)fdiv((uint32_t)rem, a.by_w);
        const int w = rem - h * a.grid_w;
        const int t = a.start_frame + (int)f;
        float2 cs[4];
        if (ROTATE) chunk_angles(cs, c8 * 4, t, h, w, a);
        const size_t src0 = (size_t)tok * a.cpt;
        size_t dst_tok = 0;  // append: chunk index of (head 0, chunk 0) of this token's cache row
        if (APPEND) {
            const int slot = t - (int)fdiv((uint32_t)t, a.by_cap) * a.cap_frames;
            dst_tok = ((size_t)slot * ft + rem) << a.cpr_log2;
        }
        for (int j0 = 0; j0 < a.cpt; j0 += 32 * kBatch) {
            uint4 xin[kBatch], vin[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int j = j0 + 32 * u + lane;
                if (j < a.cpt) {
                    xin[u] = __ldcs(a.x + src0 + j);
                    if (APPEND) vin[u] = __ldcs(a.v + src0 + j);
                }
            }
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int j = j0 + 32 * u + lane;
                if (j < a.cpt) {
                    const uint4 r = ROTATE ? rotate_chunk(xin[u], cs) : xin[u];
                    if (APPEND) {
                        const int head = j >> a.cpr_log2;
                        const size_t d = dst_tok + (((size_t)head * a.cap_tok) << a.cpr_log2) + c8;
                        __stcs(a.y + d, r);
                        __stcs(a.vc + d, vin[u]);
                    } else {
                        __stcs(a.y + src0 + j, r);
                    }
                }
            }
        }
    }
}

// SM count of the current device, looked up once per device.
int sm_count() {
    static std::mutex mu;
    static std::map<int, int> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    std::lock_guard<std::mutex> lk(mu);
    auto it = cache.find(dev);
    if (it != cache.end()) return it->second;
    int sms = 148;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) sms = 148;
    cache[dev] = sms;
    return sms;
}

// append: 0 = RoPE only, 1 = RoPE + ring write, 2 = ring write of already rotated K
int launch_stream(int append, StreamArgs& a, cudaStream_t s) {
    const long long want = ((long long)a.n_tokens + kWarpsPerBlock - 1) / kWarpsPerBlock;
    const int per_sm = append ? blocks_per_sm<true>() : blocks_per_sm<false>();
    const int blocks = (int)std::min<long long>(want, (long long)sm_count() * per_sm);
    if (blocks == 0) return VDIT_OK;
    if (append == 1)
        rope_stream_kernel<true, true><<<blocks, kWarpsPerBlock * 32, 0, s>>>(a);
    else if (append == 2)
        rope_stream_kernel<true, false><<<blocks, kWarpsPerBlock * 32, 0, s>>>(a);
    else
        rope_stream_kernel<false, true><<<blocks, kWarpsPerBlock * 32, 0, s>>>(a);
    return vdit::cuda_check(cudaGetLastError(), "rope kernel launch");
}

// Sequence-to-head pack of the Ulysses-style exchange ("Accelerating Video Generation Inference
// with Sequential-Parallel 3D Positional Encoding Using a Global Time Index", sections 2.A-2.C: the
// sequence is split over the ranks; the causal RoPE at global positions, then one fused all-to-all
// that gathers the sequence and splits the heads for Q, K and V together). Rank `rank` holds the
// chunk-local tokens rank * n_tok .. (rank + 1) * n_tok - 1 of q, k, v [n_tok, heads, D]. Block r of
// the send buffer, send [ranks][3][n_tok][heads / ranks][D], holds the heads rank r owns, Q then K
// then V; the rank's own block goes straight to rows rank * n_tok .. of its head-sharded buffers
// q_full, k_full, v_full [ranks * n_tok][heads / ranks][D], where the exchange leaves every other
// rank's block too. With ROTATE, Q and K are rotated at their global positions (the time index
// needs only start_frame and the shard's first token: no rank asks another for its positions);
// V is copied. One warp streams one (token, tensor) row.
struct PackArgs {
    StreamArgs s;       // tables, geometry, n_tokens (= n_tok), cpt, cpr_log2, start_frame
    const uint4* src[3];
    uint4* send;
    uint4* full[3];
    int rank;
    int tok0;
    int heads_per_rank;
    FastDiv by_hpr;
};

template <bool ROTATE>
__global__ void __launch_bounds__(kWarpsPerBlock * 32, 4) rope_pack_kernel(PackArgs pa) {
    const StreamArgs& a = pa.s;
    const int lane = threadIdx.x & 31;
    const int n_warps = gridDim.x * kWarpsPerBlock;
    const int c8 = lane & ((1 << a.cpr_log2) - 1);
    const int ft = a.grid_h * a.grid_w;
    const int items = 3 * a.n_tokens;
    for (int it = blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5); it < items; it += n_warps) {
        const int x = it / a.n_tokens, n = it - x * a.n_tokens;
        const bool rot = ROTATE && x < 2;
        float2 cs[4];
        if (rot) {
            const int tok = pa.tok0 + n;
            const uint32_t f = fdiv((uint32_t)tok, a.by_ft);
            const int rem = tok - (int)f * ft;
            const int h = (int)fdiv((uint32_t)rem, a.by_w);
            chunk_angles(cs, c8 * 4, a.start_frame + (int)f, h, rem - h * a.grid_w, a);
        }
        const uint4* src = pa.src[x] + (size_t)n * a.cpt;
        for (int j0 = 0; j0 < a.cpt; j0 += 32 * kBatch) {
            uint4 xin[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int j = j0 + 32 * u + lane;
                if (j < a.cpt) xin[u] = __ldcs(src + j);
            }
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int j = j0 + 32 * u + lane;
                if (j < a.cpt) {
                    const int head = j >> a.cpr_log2;
                    const int r = (int)fdiv((uint32_t)head, pa.by_hpr), hh = head - r * pa.heads_per_rank;
                    uint4* dst = r == pa.rank
                                     ? pa.full[x] + ((((size_t)pa.rank * a.n_tokens + n) * pa.heads_per_rank + hh)
                                                     << a.cpr_log2)
                                     : pa.send + (((((size_t)r * 3 + x) * a.n_tokens + n) * pa.heads_per_rank + hh)
                                                  << a.cpr_log2);
                    __stcs(dst + c8, rot ? rotate_chunk(xin[u], cs) : xin[u]);
                }
            }
        }
    }
}

// Head-to-sequence unpack after attention (the return all-to-all of the same exchange): this
// rank's tokens of out [n_tok, heads, D] gather head block r from recv[r] = [n_tok][heads /
// ranks][D] (sent by rank r, which computed those heads), block `rank` from `own` (this rank's
// own attention output rows for its tokens). A copy: bit-exact.
struct UnpackArgs {
    const uint4* recv;
    const uint4* own;
    uint4* out;
    int n_tokens, cpt, cpr_log2, rank, heads_per_rank;
    FastDiv by_hpr;
};

__global__ void __launch_bounds__(kWarpsPerBlock * 32, 4) seq_unpack_kernel(UnpackArgs a) {
    const int lane = threadIdx.x & 31;
    const int n_warps = gridDim.x * kWarpsPerBlock;
    const int c8 = lane & ((1 << a.cpr_log2) - 1);
    for (int n = blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5); n < a.n_tokens; n += n_warps) {
        for (int j0 = 0; j0 < a.cpt; j0 += 32 * kBatch) {
            uint4 xin[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int j = j0 + 32 * u + lane;
                if (j < a.cpt) {
                    const int head = j >> a.cpr_log2;
                    const int r = (int)fdiv((uint32_t)head, a.by_hpr), hh = head - r * a.heads_per_rank;
                    const uint4* src = r == a.rank
                                           ? a.own + ((((size_t)n) * a.heads_per_rank + hh) << a.cpr_log2)
                                           : a.recv + ((((size_t)r * a.n_tokens + n) * a.heads_per_rank + hh)
                                                       << a.cpr_log2);
                    xin[u] = __ldcs(src + c8);
                }
            }
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int j = j0 + 32 * u + lane;
                if (j < a.cpt) __stcs(a.out + (size_t)n * a.cpt + j, xin[u]);
            }
        }
    }
}

// The same exchange with the transfer fused into the pack: rank `rank` writes the rows of its
// tokens straight into every rank's head-sharded buffers, dst[x][r] (rank r's q_full / k_full /
// v_full, mapped into this process: peer memory over NVLink for r != rank), so the all-to-all is
// the kernel's own stores and needs no send buffer or library transfer. Each CTA ends with a
// system-scope fence: its stores are visible to the peers before the kernel completes, so a
// barrier between the ranks after the launch is all the consumers need.
struct PeerPackArgs {
    StreamArgs s;  // tables, geometry, n_tokens (= n_tok), cpt, cpr_log2, start_frame
    const uint4* src[3];
    uint4* dst[3][VDIT_MAX_PEERS];
    int rank;
    int tok0;
    int heads_per_rank;
    FastDiv by_hpr;
};

template <bool ROTATE>
__global__ void __launch_bounds__(kWarpsPerBlock * 32, 4) rope_pack_peers_kernel(PeerPackArgs pa) {
    const StreamArgs& a = pa.s;
    const int lane = threadIdx.x & 31;
    const int n_warps = gridDim.x * kWarpsPerBlock;
    const int c8 = lane & ((1 << a.cpr_log2) - 1);
    const int ft = a.grid_h * a.grid_w;
    const int items = 3 * a.n_tokens;
    for (int it = blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5); it < items; it += n_warps) {
        const int x = it / a.n_tokens, n = it - x * a.n_tokens;
        const bool rot = ROTATE && x < 2;
        float2 cs[4];
        if (rot) {
            const int tok = pa.tok0 + n;
            const uint32_t f = fdiv((uint32_t)tok, a.by_ft);
            const int rem = tok - (int)f * ft;
            const int h = (int)fdiv((uint32_t)rem, a.by_w);
            chunk_angles(cs, c8 * 4, a.start_frame + (int)f, h, rem - h * a.grid_w, a);
        }
        const uint4* src = pa.src[x] + (size_t)n * a.cpt;
        const size_t row = ((size_t)pa.rank * a.n_tokens + n) * pa.heads_per_rank;
        for (int j0 = 0; j0 < a.cpt; j0 += 32 * kBatch) {
            uint4 xin[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int j = j0 + 32 * u + lane;
                if (j < a.cpt) xin[u] = __ldcs(src + j);
            }
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int j = j0 + 32 * u + lane;
                if (j < a.cpt) {
                    const int head = j >> a.cpr_log2;
                    const int r = (int)fdiv((uint32_t)head, pa.by_hpr), hh = head - r * pa.heads_per_rank;
                    uint4* dst = pa.dst[x][r] + ((row + hh) << a.cpr_log2);
                    __stcs(dst + c8, rot ? rotate_chunk(xin[u], cs) : xin[u]);
                }
            }
        }
    }
    __threadfence_system();
}

// Push form of the return exchange: this rank holds o_full [ranks * n_tok][heads / ranks][D], its
// heads' attention output for every rank's tokens, and writes the rows of rank s's tokens into
// rank s's output out_dst[s] [n_tok][heads][D] at this rank's head columns (peer memory for
// s != rank). A copy: bit-exact. System-scope fence at the end, as above.
struct PeerPushArgs {
    const uint4* o_full;
    uint4* dst[VDIT_MAX_PEERS];
    int n_tokens, n_ranks, rank, row_chunks, cpt;  // row_chunks: (heads / ranks) * D / 8
    FastDiv by_ntok;
};

__global__ void __launch_bounds__(kWarpsPerBlock * 32, 4) seq_push_peers_kernel(PeerPushArgs a) {
    const int lane = threadIdx.x & 31;
    const int n_warps = gridDim.x * kWarpsPerBlock;
    const int rows = a.n_ranks * a.n_tokens;
    for (int it = blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5); it < rows; it += n_warps) {
        const int s = (int)fdiv((uint32_t)it, a.by_ntok), n = it - s * a.n_tokens;
        const uint4* src = a.o_full + (size_t)it * a.row_chunks;
        uint4* dst = a.dst[s] + (size_t)n * a.cpt + (size_t)a.rank * a.row_chunks;
        for (int j0 = 0; j0 < a.row_chunks; j0 += 32 * kBatch) {
            uint4 xin[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int j = j0 + 32 * u + lane;
                if (j < a.row_chunks) xin[u] = __ldcs(src + j);
            }
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int j = j0 + 32 * u + lane;
                if (j < a.row_chunks) __stcs(dst + j, xin[u]);
            }
        }
    }
    __threadfence_system();
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int fill_common(const vdit_geom* g, StreamArgs& a) {
    vdit::RopeTables tabs;
    if (int rc = vdit::get_rope_tables(g, &tabs)) return rc;
    a.tt = static_cast<const float2*>(tabs.t);
    a.th = static_cast<const float2*>(tabs.h);
    a.tw = static_cast<const float2*>(tabs.w);
    a.bt2 = g->band_t / 2;
    a.bh2 = g->band_h / 2;
    a.bw2 = g->band_w / 2;
    a.cpr_log2 = g->head_dim == 128 ? 4 : 3;
    a.cpt = g->heads * (g->head_dim / 8);
    a.grid_h = g->grid_h;
    a.grid_w = g->grid_w;
    a.by_ft = make_fastdiv((uint32_t)(g->grid_h * g->grid_w));
    a.by_w = make_fastdiv((uint32_t)g->grid_w);
    a.by_cap = make_fastdiv(1);
    return VDIT_OK;
}

}  // namespace

extern "C" int vdit_rope3d_apply(const vdit_geom* g, const void* x, void* y, int start_frame,
                                 long long n_tokens, void* stream) {
    using vdit::fail;
    if (int rc = vdit::check_geom(g)) return rc;
    if (n_tokens < 0) return fail(VDIT_ERR_INVALID_ARG, "n_tokens < 0");
    if (n_tokens == 0) return VDIT_OK;
    if (!x || !y) return fail(VDIT_ERR_INVALID_ARG, "x or y is NULL");
    if (!aligned16(x) || !aligned16(y)) return fail(VDIT_ERR_MISALIGNED, "x/y not 16-byte aligned");
    const long long ft = (long long)g->grid_h * g->grid_w;
    const long long frames = (n_tokens + ft - 1) / ft;
    if (start_frame < 0 || start_frame + frames - 1 > VDIT_MAX_FRAME)
        return fail(VDIT_ERR_INVALID_ARG, "frames outside [0, VDIT_MAX_FRAME]");
    const long long row_bytes = (long long)g->heads * g->head_dim * 2;
    const char* xb = static_cast<const char*>(x);
    char* yb = static_cast<char*>(y);
    if (xb != yb && xb < yb + n_tokens * row_bytes && yb < xb + n_tokens * row_bytes)
        return fail(VDIT_ERR_INVALID_ARG, "x and y overlap without being identical");
    if ((unsigned long long)n_tokens * g->heads * (g->head_dim / 8) >= (1ull << 31))
        return fail(VDIT_ERR_UNSUPPORTED, "tensor larger than 2^31 16-byte chunks (32 GiB)");
    StreamArgs a{};
    if (int rc = fill_common(g, a)) return rc;
    a.x = static_cast<const uint4*>(x);
    a.y = static_cast<uint4*>(y);
    a.n_tokens = (int)n_tokens;
    a.start_frame = start_frame;
    return launch_stream(0, a, static_cast<cudaStream_t>(stream));
}

namespace {
int kv_ring_write(const vdit_geom* g, void* k_cache, void* v_cache, int capacity_frames, const void* k,
                  const void* v, int start_frame, int n_frames, bool rotate, void* stream) {
    using vdit::fail;
    if (int rc = vdit::check_geom(g)) return rc;
    if (!k_cache || !v_cache || !k || !v) return fail(VDIT_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k) || !aligned16(v))
        return fail(VDIT_ERR_MISALIGNED, "tensor not 16-byte aligned");
    if (capacity_frames < 1 || n_frames < 1 || n_frames > capacity_frames)
        return fail(VDIT_ERR_INVALID_ARG, "need 1 <= n_frames <= capacity_frames");
    if (start_frame < 0 || start_frame + n_frames - 1 > VDIT_MAX_FRAME)
        return fail(VDIT_ERR_INVALID_ARG, "frames outside [0, VDIT_MAX_FRAME]");
    const long long ft = (long long)g->grid_h * g->grid_w;
    const long long row = (long long)g->heads * g->head_dim * 2;
    const long long chunk_bytes = ft * n_frames * row, cache_bytes = ft * capacity_frames * row;
    auto overlap = [](const void* a, long long na, const void* b, long long nb) {
        const char* x = static_cast<const char*>(a);
        const char* y = static_cast<const char*>(b);
        return x < y + nb && y < x + na;
    };
    if (overlap(k_cache, cache_bytes, v_cache, cache_bytes) ||
        overlap(k_cache, cache_bytes, k, chunk_bytes) || overlap(k_cache, cache_bytes, v, chunk_bytes) ||
        overlap(v_cache, cache_bytes, k, chunk_bytes) || overlap(v_cache, cache_bytes, v, chunk_bytes))
        return fail(VDIT_ERR_INVALID_ARG, "caches overlap each other or the chunk");
    if ((unsigned long long)chunk_bytes / 16 >= (1ull << 31))
        return fail(VDIT_ERR_UNSUPPORTED, "chunk larger than 2^31 16-byte chunks (32 GiB)");
    StreamArgs a{};
    if (int rc = fill_common(g, a)) return rc;
    a.x = static_cast<const uint4*>(k);
    a.v = static_cast<const uint4*>(v);
    a.y = static_cast<uint4*>(k_cache);
    a.vc = static_cast<uint4*>(v_cache);
    a.n_tokens = (int)(ft * n_frames);
    a.start_frame = start_frame;
    a.cap_frames = capacity_frames;
    a.cap_tok = ft * capacity_frames;
    a.by_cap = make_fastdiv((uint32_t)capacity_frames);
    return launch_stream(rotate ? 1 : 2, a, static_cast<cudaStream_t>(stream));
}
}  // namespace

extern "C" int vdit_kv_append(const vdit_geom* g, void* k_cache, void* v_cache,
                              int capacity_frames, const void* k, const void* v, int start_frame,
                              int n_frames, void* stream) {
    return kv_ring_write(g, k_cache, v_cache, capacity_frames, k, v, start_frame, n_frames, true, stream);
}

extern "C" int vdit_kv_write(const vdit_geom* g, void* k_cache, void* v_cache, int capacity_frames,
                             const void* k_rotated, const void* v, int start_frame, int n_frames,
                             void* stream) {
    return kv_ring_write(g, k_cache, v_cache, capacity_frames, k_rotated, v, start_frame, n_frames, false,
                         stream);
}

extern "C" int vdit_seq_pack(const vdit_geom* g, const void* q, const void* k, const void* v, void* send,
                             void* q_full, void* k_full, void* v_full, int rank, int n_ranks, int start_frame,
                             long long n_tokens, int rotate, void* stream) {
    using vdit::fail;
    if (int rc = vdit::check_geom(g)) return rc;
    if (n_tokens < 0) return fail(VDIT_ERR_INVALID_ARG, "n_tokens must be >= 0");
    if (n_ranks < 1 || g->heads % n_ranks != 0) return fail(VDIT_ERR_INVALID_ARG, "n_ranks must divide heads");
    if (rank < 0 || rank >= n_ranks) return fail(VDIT_ERR_INVALID_ARG, "rank outside [0, n_ranks)");
    if (n_tokens == 0) return VDIT_OK;
    if (!q || !k || !v || !q_full || !k_full || !v_full || (n_ranks > 1 && !send))
        return fail(VDIT_ERR_INVALID_ARG, "NULL pointer");
    const void* ptrs[7] = {q, k, v, send, q_full, k_full, v_full};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return fail(VDIT_ERR_MISALIGNED, "tensor not 16-byte aligned");
    const long long ft = (long long)g->grid_h * g->grid_w;
    const long long tok0 = (long long)rank * n_tokens, last = tok0 + n_tokens - 1;
    if (start_frame < 0 || start_frame + last / ft > VDIT_MAX_FRAME)
        return fail(VDIT_ERR_INVALID_ARG, "frames outside [0, VDIT_MAX_FRAME]");
    if ((unsigned long long)n_tokens * n_ranks * g->heads * (g->head_dim / 8) >= (1ull << 31) ||
        (long long)n_tokens * n_ranks >= (1ll << 31))
        return fail(VDIT_ERR_UNSUPPORTED, "exchange larger than 2^31 16-byte chunks");
    // inputs (3 x n_tokens rows) against outputs (send: 3 x n_ranks x n_tokens rows; each full
    // buffer: n_ranks x n_tokens rows of heads / n_ranks heads) must not overlap
    const long long in_bytes = n_tokens * g->heads * g->head_dim * 2;
    const long long full_bytes = in_bytes;  // n_ranks * n_tokens * (heads / n_ranks) * D * 2
    const long long send_bytes = 3 * in_bytes;
    const void* outs[4] = {send, q_full, k_full, v_full};
    const long long out_n[4] = {n_ranks > 1 ? send_bytes : 0, full_bytes, full_bytes, full_bytes};
    auto overlap = [](const void* a, long long na, const void* b, long long nb) {
        const char* x = static_cast<const char*>(a);
        const char* y = static_cast<const char*>(b);
        return na > 0 && nb > 0 && x < y + nb && y < x + na;
    };
    for (int i = 0; i < 4; ++i) {
        for (int j = 0; j < 3; ++j)
            if (overlap(outs[i], out_n[i], ptrs[j], in_bytes))
                return fail(VDIT_ERR_INVALID_ARG, "an output overlaps an input");
        for (int j = i + 1; j < 4; ++j)
            if (overlap(outs[i], out_n[i], outs[j], out_n[j]))
                return fail(VDIT_ERR_INVALID_ARG, "outputs overlap each other");
    }
    PackArgs pa{};
    if (int rc = fill_common(g, pa.s)) return rc;
    pa.s.n_tokens = (int)n_tokens;
    pa.s.start_frame = start_frame;
    pa.src[0] = static_cast<const uint4*>(q);
    pa.src[1] = static_cast<const uint4*>(k);
    pa.src[2] = static_cast<const uint4*>(v);
    pa.send = static_cast<uint4*>(send);
    pa.full[0] = static_cast<uint4*>(q_full);
    pa.full[1] = static_cast<uint4*>(k_full);
    pa.full[2] = static_cast<uint4*>(v_full);
    pa.rank = rank;
    pa.tok0 = (int)tok0;
    pa.heads_per_rank = g->heads / n_ranks;
    pa.by_hpr = make_fastdiv((uint32_t)pa.heads_per_rank);
    const long long want = (3 * n_tokens + kWarpsPerBlock - 1) / kWarpsPerBlock;
    const int blocks = (int)std::min<long long>(want, (long long)sm_count() * 4);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (rotate)
        rope_pack_kernel<true><<<blocks, kWarpsPerBlock * 32, 0, st>>>(pa);
    else
        rope_pack_kernel<false><<<blocks, kWarpsPerBlock * 32, 0, st>>>(pa);
    return vdit::cuda_check(cudaGetLastError(), "pack kernel launch");
}

extern "C" int vdit_seq_unpack(const vdit_geom* g, const void* recv, const void* own, void* out, int rank,
                               int n_ranks, long long n_tokens, void* stream) {
    using vdit::fail;
    if (int rc = vdit::check_geom(g)) return rc;
    if (n_tokens < 0) return fail(VDIT_ERR_INVALID_ARG, "n_tokens must be >= 0");
    if (n_ranks < 1 || g->heads % n_ranks != 0) return fail(VDIT_ERR_INVALID_ARG, "n_ranks must divide heads");
    if (rank < 0 || rank >= n_ranks) return fail(VDIT_ERR_INVALID_ARG, "rank outside [0, n_ranks)");
    if (n_tokens == 0) return VDIT_OK;
    if (!own || !out || (n_ranks > 1 && !recv)) return fail(VDIT_ERR_INVALID_ARG, "NULL pointer");
    if ((recv && !aligned16(recv)) || !aligned16(own) || !aligned16(out))
        return fail(VDIT_ERR_MISALIGNED, "tensor not 16-byte aligned");
    const long long out_bytes = n_tokens * g->heads * g->head_dim * 2;
    const long long own_bytes = out_bytes / n_ranks, recv_bytes = n_ranks > 1 ? out_bytes : 0;
    auto overlap = [](const void* a, long long na, const void* b, long long nb) {
        const char* x = static_cast<const char*>(a);
        const char* y = static_cast<const char*>(b);
        return na > 0 && nb > 0 && x < y + nb && y < x + na;
    };
    if (overlap(out, out_bytes, own, own_bytes) || overlap(out, out_bytes, recv, recv_bytes))
        return fail(VDIT_ERR_INVALID_ARG, "out overlaps an input");
    if ((unsigned long long)n_tokens * g->heads * (g->head_dim / 8) >= (1ull << 31))
        return fail(VDIT_ERR_UNSUPPORTED, "shard larger than 2^31 16-byte chunks");
    UnpackArgs a{};
    a.recv = static_cast<const uint4*>(recv);
    a.own = static_cast<const uint4*>(own);
    a.out = static_cast<uint4*>(out);
    a.n_tokens = (int)n_tokens;
    a.cpr_log2 = g->head_dim == 128 ? 4 : 3;
    a.cpt = g->heads * (g->head_dim / 8);
    a.rank = rank;
    a.heads_per_rank = g->heads / n_ranks;
    a.by_hpr = make_fastdiv((uint32_t)a.heads_per_rank);
    const long long want = (n_tokens + kWarpsPerBlock - 1) / kWarpsPerBlock;
    const int blocks = (int)std::min<long long>(want, (long long)sm_count() * 4);
    seq_unpack_kernel<<<blocks, kWarpsPerBlock * 32, 0, static_cast<cudaStream_t>(stream)>>>(a);
    return vdit::cuda_check(cudaGetLastError(), "unpack kernel launch");
}

extern "C" int vdit_seq_pack_peers(const vdit_geom* g, const void* q, const void* k, const void* v,
                                   void* const* q_dst, void* const* k_dst, void* const* v_dst, int rank,
                                   int n_ranks, int start_frame, long long n_tokens, int rotate, void* stream) {
    using vdit::fail;
    if (int rc = vdit::check_geom(g)) return rc;
    if (n_tokens < 0) return fail(VDIT_ERR_INVALID_ARG, "n_tokens must be >= 0");
    if (n_ranks < 1 || n_ranks > VDIT_MAX_PEERS || g->heads % n_ranks != 0)
        return fail(VDIT_ERR_INVALID_ARG, "n_ranks must divide heads and be at most VDIT_MAX_PEERS");
    if (rank < 0 || rank >= n_ranks) return fail(VDIT_ERR_INVALID_ARG, "rank outside [0, n_ranks)");
    if (n_tokens == 0) return VDIT_OK;
    if (!q || !k || !v || !q_dst || !k_dst || !v_dst) return fail(VDIT_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return fail(VDIT_ERR_MISALIGNED, "input not 16-byte aligned");
    for (int r = 0; r < n_ranks; ++r) {
        if (!q_dst[r] || !k_dst[r] || !v_dst[r]) return fail(VDIT_ERR_INVALID_ARG, "NULL destination");
        if (!aligned16(q_dst[r]) || !aligned16(k_dst[r]) || !aligned16(v_dst[r]))
            return fail(VDIT_ERR_MISALIGNED, "destination not 16-byte aligned");
    }
    const long long ft = (long long)g->grid_h * g->grid_w;
    const long long tok0 = (long long)rank * n_tokens, last = tok0 + n_tokens - 1;
    if (start_frame < 0 || start_frame + last / ft > VDIT_MAX_FRAME)
        return fail(VDIT_ERR_INVALID_ARG, "frames outside [0, VDIT_MAX_FRAME]");
    if ((unsigned long long)n_tokens * n_ranks * g->heads * (g->head_dim / 8) >= (1ull << 31) ||
        (long long)n_tokens * n_ranks >= (1ll << 31))
        return fail(VDIT_ERR_UNSUPPORTED, "exchange larger than 2^31 16-byte chunks");
    // this rank's own head-sharded buffers (the only destinations in this address space that the
    // call can tell apart from peer mappings) must not overlap the inputs or one another
    const long long in_bytes = n_tokens * g->heads * g->head_dim * 2;
    const long long full_bytes = in_bytes;  // n_ranks * n_tokens * (heads / n_ranks) * D * 2
    const void* ins[3] = {q, k, v};
    const void* own[3] = {q_dst[rank], k_dst[rank], v_dst[rank]};
    auto overlap = [](const void* a, long long na, const void* b, long long nb) {
        const char* x = static_cast<const char*>(a);
        const char* y = static_cast<const char*>(b);
        return x < y + nb && y < x + na;
    };
    for (int i = 0; i < 3; ++i) {
        for (int j = 0; j < 3; ++j)
            if (overlap(own[i], full_bytes, ins[j], in_bytes))
                return fail(VDIT_ERR_INVALID_ARG, "an output overlaps an input");
        for (int j = i + 1; j < 3; ++j)
            if (overlap(own[i], full_bytes, own[j], full_bytes))
                return fail(VDIT_ERR_INVALID_ARG, "outputs overlap each other");
    }
    PeerPackArgs pa{};
    if (int rc = fill_common(g, pa.s)) return rc;
    pa.s.n_tokens = (int)n_tokens;
    pa.s.start_frame = start_frame;
    pa.src[0] = static_cast<const uint4*>(q);
    pa.src[1] = static_cast<const uint4*>(k);
    pa.src[2] = static_cast<const uint4*>(v);
    void* const* dsts[3] = {q_dst, k_dst, v_dst};
    for (int x = 0; x < 3; ++x)
        for (int r = 0; r < n_ranks; ++r) pa.dst[x][r] = static_cast<uint4*>(dsts[x][r]);
    pa.rank = rank;
    pa.tok0 = (int)tok0;
    pa.heads_per_rank = g->heads / n_ranks;
    pa.by_hpr = make_fastdiv((uint32_t)pa.heads_per_rank);
    const long long want = (3 * n_tokens + kWarpsPerBlock - 1) / kWarpsPerBlock;
    const int blocks = (int)std::min<long long>(want, (long long)sm_count() * 4);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (rotate)
        rope_pack_peers_kernel<true><<<blocks, kWarpsPerBlock * 32, 0, st>>>(pa);
    else
        rope_pack_peers_kernel<false><<<blocks, kWarpsPerBlock * 32, 0, st>>>(pa);
    return vdit::cuda_check(cudaGetLastError(), "peer pack kernel launch");
}

extern "C" int vdit_seq_push_peers(const vdit_geom* g, const void* o_full, void* const* out_dst, int rank,
                                   int n_ranks, long long n_tokens, void* stream) {
    using vdit::fail;
    if (int rc = vdit::check_geom(g)) return rc;
    if (n_tokens < 0) return fail(VDIT_ERR_INVALID_ARG, "n_tokens must be >= 0");
    if (n_ranks < 1 || n_ranks > VDIT_MAX_PEERS || g->heads % n_ranks != 0)
        return fail(VDIT_ERR_INVALID_ARG, "n_ranks must divide heads and be at most VDIT_MAX_PEERS");
    if (rank < 0 || rank >= n_ranks) return fail(VDIT_ERR_INVALID_ARG, "rank outside [0, n_ranks)");
    if (n_tokens == 0) return VDIT_OK;
    if (!o_full || !out_dst) return fail(VDIT_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned16(o_full)) return fail(VDIT_ERR_MISALIGNED, "o_full not 16-byte aligned");
    for (int r = 0; r < n_ranks; ++r) {
        if (!out_dst[r]) return fail(VDIT_ERR_INVALID_ARG, "NULL destination");
        if (!aligned16(out_dst[r])) return fail(VDIT_ERR_MISALIGNED, "destination not 16-byte aligned");
    }
    const long long out_bytes = n_tokens * g->heads * g->head_dim * 2;
    const long long in_bytes = out_bytes;  // n_ranks * n_tokens * (heads / n_ranks) * D * 2
    const char* x = static_cast<const char*>(o_full);
    const char* y = static_cast<const char*>(out_dst[rank]);
    if (x < y + out_bytes && y < x + in_bytes) return fail(VDIT_ERR_INVALID_ARG, "output overlaps o_full");
    if ((unsigned long long)n_tokens * n_ranks * g->heads * (g->head_dim / 8) >= (1ull << 31) ||
        (long long)n_tokens * n_ranks >= (1ll << 31))
        return fail(VDIT_ERR_UNSUPPORTED, "exchange larger than 2^31 16-byte chunks");
    PeerPushArgs a{};
    a.o_full = static_cast<const uint4*>(o_full);
    for (int r = 0; r < n_ranks; ++r) a.dst[r] = static_cast<uint4*>(out_dst[r]);
    a.n_tokens = (int)n_tokens;
    a.n_ranks = n_ranks;
    a.rank = rank;
    a.row_chunks = (g->heads / n_ranks) * (g->head_dim / 8);
    a.cpt = g->heads * (g->head_dim / 8);
    a.by_ntok = make_fastdiv((uint32_t)n_tokens);
    const long long want = ((long long)n_ranks * n_tokens + kWarpsPerBlock - 1) / kWarpsPerBlock;
    const int blocks = (int)std::min<long long>(want, (long long)sm_count() * 4);
    seq_push_peers_kernel<<<blocks, kWarpsPerBlock * 32, 0, static_cast<cudaStream_t>(stream)>>>(a);
    return vdit::cuda_check(cudaGetLastError(), "peer push kernel launch");
}
