// Fused QKV projection + 3-D RoPE + KV-cache append on tcgen05 tensor cores (libvdit, sm_100a).
//
// "Accelerating Video Generation Inference with Sequential-Parallel 3D Positional Encoding Using
// a Global Time Index", section 2.C, fuses the QKV projections and the causal RoPE into one
// kernel; section 2.B gives each chunk global temporal positions t = start_frame + local frame;
// section 2.A keeps K and V of past chunks in a cache. Here one persistent GEMM computes
//   [Q | K | V] = X W^T        (X [tokens, d_model], W [3 * heads * head_dim, d_model], bf16)
// in fp32 on the tensor cores and its epilogue rotates Q and K at the tokens' global positions
// (fp32 math, tables built in fp64) and stores bf16: Q to [tokens, heads, head_dim], K' and V
// straight into the chunk's frame slots of the head-major ring cache (what vdit_kv_append does).
//
// One CTA per SM, persistent over 128 x 256 output tiles (in the order that keeps the smaller
// operand in L2); 6 warps:
//   warp 0      producer: TMA (SWIZZLE_128B) of the 128 x 64 X tile and the 256 x 64 W tile of
//               each 64-wide k step into a 4-stage ring;
//   warp 1      TMEM allocator (512 columns: two 256-column fp32 accumulators) and the single
//               thread issuing kind::f16 MMAs, M = 128, N = 256, K = 16 (four per k step);
//   warps 2-5   epilogue: thread r owns accumulator row r (TMEM lane r); per 64-column slab it
//               loads the fp32 row (tcgen05.ld), rotates the pairs, rounds to bf16 into a
//               swizzled shared-memory slab and one thread stores the slab with a TMA tensor
//               store. The accumulator is released as soon as it has been read, so the next
//               tile's MMAs overlap the stores.
// Every mbarrier wait is bounded (globaltimer); on expiry the CTA raises its abort flag and the
// status word (VDIT_ERR_TIMEOUT), drains what it issued and frees TMEM before exiting.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "sm100.h"

namespace {

constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kGStages = 4;
constexpr int kGThreads = 192;
constexpr int kGWarpTMA = 0, kGWarpMMA = 1;  // warps 2-5: epilogue
constexpr uint32_t kABytes = kBM * kBK * 2;        // 16 KiB
constexpr uint32_t kBBytes = kBN * kBK * 2;        // 32 KiB
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr uint32_t kOutSlab = kBM * 64 * 2;        // 16 KiB: 128 rows x 64 columns of bf16
constexpr uint32_t kAccCols = kBN;                 // fp32 columns per accumulator

enum { G_FULL = 0, G_EMPTY = G_FULL + kGStages, G_AFULL = G_EMPTY + kGStages,
       G_AEMPTY = G_AFULL + 2, G_DRAIN = G_AEMPTY + 2, G_COUNT };
static_assert(G_COUNT <= 16, "barrier area");

constexpr uint32_t OFF_STAGE = 0;
constexpr uint32_t OFF_OUT = OFF_STAGE + kGStages * kStageBytes;     // two output slabs
constexpr uint32_t OFF_BAR = OFF_OUT + 2 * kOutSlab;
constexpr uint32_t OFF_MISC = OFF_BAR + 8 * 16;                        // [0] tmem, [1] abort
constexpr uint32_t kGSmemBytes = OFF_MISC + 64 + 1024;                 // + alignment slack
static_assert(kGSmemBytes <= 227 * 1024, "shared memory budget");

struct GemmArgs {
    int m;              // tokens of this launch
    int k;              // d_model
    int n_tiles_m, n_tiles_n;
    int n_major;        // tile order: 0 = row blocks outer (W stays in L2), 1 = column blocks outer
    int hd;             // heads * head_dim (one of the Q, K, V sections)
    int head_dim;
    int tok0;           // chunk-local index of this launch's first token
    int start_frame;    // global frame of the chunk's first token
    int grid_h, grid_w;
    const float2* tt;
    const float2* th;
    const float2* tw;
    int bt2, bh2, bw2;
    int* status;
};

__device__ int g_qkv_status = 0;

// Output tile t -> (first row, first column). Consecutive tiles run at the same time on different
// SMs, so the operand they share should be the one that does not fit in L2: with row blocks
// outer they share X rows and stream all of W (kept when W is the smaller), with column blocks
// outer they share W columns and stream all of X.
__device__ __forceinline__ void tile_origin(int t, const GemmArgs& a, int& m0, int& n0) {
    if (a.n_major) {
        m0 = (t % a.n_tiles_m) * kBM;
        n0 = (t / a.n_tiles_m) * kBN;
    } else {
        m0 = (t / a.n_tiles_n) * kBM;
        n0 = (t % a.n_tiles_n) * kBN;
    }
}

// (cos, sin) of RoPE pair pp of a head vector at position (t, h, w): bands t, h, w in order.
__device__ __forceinline__ float2 pair_angle(int pp, int t, int h, int w, const GemmArgs& a) {
    const bool in_h = pp >= a.bt2, in_w = pp >= a.bt2 + a.bh2;
    const float2* tab = in_w ? a.tw : (in_h ? a.th : a.tt);
    const int row = in_w ? w : (in_h ? h : t);
    const int width = in_w ? a.bw2 : (in_h ? a.bh2 : a.bt2);
    const int jj = pp - (in_w ? a.bt2 + a.bh2 : (in_h ? a.bt2 : 0));
    return __ldg(tab + (size_t)row * width + jj);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(map), "r"(bar), "r"(c0), "r"(c1)
        : "memory");
}
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int c0, int c1) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(map),
                 "r"(src), "r"(c0), "r"(c1)
                 : "memory");
}
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, uint32_t src, int c0, int c1, int c2) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(map),
                 "r"(src), "r"(c0), "r"(c1), "r"(c2)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Waits until at most n committed bulk groups of this thread still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__global__ void __launch_bounds__(kGThreads, 1)
    qkv_rope_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
                    const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                    const __grid_constant__ CUtensorMap map_v, const GemmArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    auto BAR = [&](int i) { return sbase + OFF_BAR + 8u * (uint32_t)i; };
    volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(smem + OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_tiles = a.n_tiles_m * a.n_tiles_n;
    const int k_steps = (a.k + kBK - 1) / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGStages; ++s) {
            mbar_init(BAR(G_FULL + s), 1);
            mbar_init(BAR(G_EMPTY + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(BAR(G_AFULL + b), 1);
            mbar_init(BAR(G_AEMPTY + b), 128);
        }
        mbar_init(BAR(G_DRAIN), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kGWarpMMA) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(sbase + OFF_MISC),
                     "r"(2 * kAccCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];

    if (warp == kGWarpTMA) {
        // ---------------------------------------------------------------------- producer
        int it = 0, issued = 0;
        bool ok = true;
        for (int tile = blockIdx.x; ok && tile < n_tiles; tile += gridDim.x) {
            int m0, n0;
            tile_origin(tile, a, m0, n0);
            for (int ks = 0; ks < k_steps; ++ks, ++it) {
                const int s = it % kGStages;
                if (it >= kGStages &&
                    !warp_wait(BAR(G_EMPTY + s), (uint32_t)((it / kGStages) - 1) & 1u, abort_flag, a.status)) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    mbar_expect_tx(BAR(G_FULL + s), kStageBytes);
                    const uint32_t dst = sbase + OFF_STAGE + s * kStageBytes;
                    tma_load_2d(dst, &map_x, BAR(G_FULL + s), ks * kBK, m0);
                    tma_load_2d(dst + kABytes, &map_w, BAR(G_FULL + s), ks * kBK, n0);
                }
                issued = it + 1;
                __syncwarp();
            }
        }
        if (*abort_flag && lane == 0) {
            // drain: the last kGStages loads this warp issued must land before the CTA exits
            for (int i = max(0, issued - kGStages); i < issued; ++i) {
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait(BAR(G_FULL + i % kGStages), (uint32_t)(i / kGStages) & 1u) &&
                       globaltimer() - t0 < kWaitLimitNs) {
                }
            }
        }
    } else if (warp == kGWarpMMA) {
        // ---------------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = instr_desc(kBN, 0);
            const uint64_t da = smem_desc_sw128(sbase + OFF_STAGE, 16, 1024);
            const uint64_t db = smem_desc_sw128(sbase + OFF_STAGE + kABytes, 16, 1024);
            constexpr uint64_t kStageDesc = kStageBytes >> 4;
            int it = 0, nt = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < n_tiles; tile += gridDim.x, ++nt) {
                const int b = nt & 1;
                if (nt >= 2) {  // the epilogue has read this accumulator's previous tile
                    if (!wait_bounded(BAR(G_AEMPTY + b), (uint32_t)((nt >> 1) - 1) & 1u, abort_flag, a.status)) break;
                    tc_fence_after();
                }
                const uint32_t d_t = tmem + (uint32_t)b * kAccCols;
                for (int ks = 0; ks < k_steps; ++ks, ++it) {
                    const int s = it % kGStages;
                    if (!wait_bounded(BAR(G_FULL + s), (uint32_t)(it / kGStages) & 1u, abort_flag, a.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t sa = da + (uint64_t)s * kStageDesc, sb = db + (uint64_t)s * kStageDesc;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        tc_mma(d_t, sa + (uint64_t)(kk * 2), sb + (uint64_t)(kk * 2), idesc, (ks | kk) ? 1u : 0u);
                    tc_commit(BAR(G_EMPTY + s));
                }
                if (!ok) break;
                tc_commit(BAR(G_AFULL + b));
            }
            tc_commit(BAR(G_DRAIN));
            const uint64_t t0 = globaltimer();
            while (!mbar_try_wait(BAR(G_DRAIN), 0) && globaltimer() - t0 < kWaitLimitNs) {
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------------- epilogue
        const int row = (warp & 3) * 32 + lane;  // TMEM lane of this warp's quarter
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const bool leader = threadIdx.x == 64;   // issues the TMA stores
        const int ft = a.grid_h * a.grid_w;
        int nt = 0, slab_n = 0;
        for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++nt) {
            const int b = nt & 1;
            int m0, n0;
            tile_origin(tile, a, m0, n0);
            // the four epilogue warps decide together, so none is left alone in a named barrier
            const bool got = warp_wait(BAR(G_AFULL + b), (uint32_t)(nt >> 1) & 1u, abort_flag, a.status);
            uint32_t all_got;
            asm volatile(
                "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
                "bar.red.and.pred q, 1, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
                : "=r"(all_got)
                : "r"((uint32_t)got)
                : "memory");
            if (!all_got) break;
            tc_fence_after();
            const int section = n0 / a.hd;             // 0: Q, 1: K, 2: V
            const int col0 = n0 - section * a.hd;      // first feature of the tile in its section
            // position of this row's token (rows past the launch's tokens are never stored)
            const int tok = a.tok0 + min(m0 + row, a.m - 1);
            const int f = tok / ft, rem = tok - f * ft;
            const int t = a.start_frame + f, hh = rem / a.grid_w, ww = rem - hh * a.grid_w;
            for (int sl = 0; sl < kBN / 64; ++sl, ++slab_n) {
                uint32_t v[64];
                tmem_ld32(tmem + lane_base + (uint32_t)b * kAccCols + sl * 64, v);
                tmem_ld32(tmem + lane_base + (uint32_t)b * kAccCols + sl * 64 + 32, v + 32);
                tmem_ld_wait(v);
                reg_touch32(v + 32);
                if (sl == kBN / 64 - 1) {
                    // every column of the accumulator is in registers: release it to the MMAs
                    tc_fence_before();
                    mbar_arrive(BAR(G_AEMPTY + b));
                }
                const int feat0 = col0 + sl * 64;  // first feature of the slab in its section
                if (section < 2) {
                    const int pp0 = (feat0 % a.head_dim) >> 1;  // first pair of the slab in its head
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const float2 cs = pair_angle(pp0 + i, t, hh, ww, a);
                        const float x0 = __uint_as_float(v[2 * i]), x1 = __uint_as_float(v[2 * i + 1]);
                        v[2 * i] = __float_as_uint(fmaf(x0, cs.x, -x1 * cs.y));
                        v[2 * i + 1] = __float_as_uint(fmaf(x0, cs.y, x1 * cs.x));
                    }
                }
                // the staging slab written two slabs ago must have been read by its TMA store
                const int buf = slab_n & 1;
                if (leader) bulk_wait_read<1>();
                asm volatile("bar.sync 1, 128;" ::: "memory");
                uint8_t* stage = smem + OFF_OUT + buf * kOutSlab;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint32_t w4[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        __nv_bfloat162 p2 = __floats2bfloat162_rn(__uint_as_float(v[8 * c + 2 * e]),
                                                                  __uint_as_float(v[8 * c + 2 * e + 1]));
                        memcpy(&w4[e], &p2, 4);
                    }
                    *reinterpret_cast<uint4*>(stage + row * 128 + ((c ^ (row & 7)) << 4)) =
                        make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
                fence_proxy_async_smem();
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (leader) {
                    const uint32_t src = sbase + OFF_OUT + buf * kOutSlab;
                    if (section == 0)
                        tma_store_2d(&map_q, src, feat0, m0);
                    else
                        tma_store_3d(section == 1 ? &map_k : &map_v, src, feat0 % a.head_dim, m0,
                                     feat0 / a.head_dim);
                    bulk_commit();
                }
            }
        }
        if (leader) bulk_wait_all();
    }
    // ------------------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == kGWarpMMA) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * kAccCols)
                     : "memory");
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// bf16 tensor map with the 128-byte swizzle; dims[0] innermost (elements), strides in bytes for
// dims 1.. ; box[0] = 64 elements (128 bytes).
int encode(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
           const cuuint32_t* box) {
    auto enc = encoder();
    if (!enc) return vdit::fail(VDIT_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides,
                           box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? VDIT_OK : vdit::fail(VDIT_ERR_CUDA, "cuTensorMapEncodeTiled failed");
}

// Per-device set-up, once per device with that device current: the kernel's dynamic shared-memory
// opt-in (a function attribute belongs to one device's context), the status word's device
// address and the SM count.
struct QkvDeviceState {
    bool ready = false;
    int* status = nullptr;
    int sms = 148;
};
constexpr int kMaxDevices = 256;
std::mutex g_qkv_dev_mu;
QkvDeviceState g_qkv_dev[kMaxDevices];

int qkv_device_state(int dev, QkvDeviceState* out) {
    if (dev < 0 || dev >= kMaxDevices) return vdit::fail(VDIT_ERR_INVALID_ARG, "device index too large");
    std::lock_guard<std::mutex> lk(g_qkv_dev_mu);
    QkvDeviceState& st = g_qkv_dev[dev];
    if (!st.ready) {
        if (int rc = vdit::cuda_check(cudaFuncSetAttribute(qkv_rope_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                           (int)kGSmemBytes),
                                      "cudaFuncSetAttribute(qkv_rope)"))
            return rc;
        void* sp = nullptr;
        if (int rc = vdit::cuda_check(cudaGetSymbolAddress(&sp, g_qkv_status), "cudaGetSymbolAddress(status)"))
            return rc;
        st.status = static_cast<int*>(sp);
        if (int rc = vdit::cuda_check(cudaDeviceGetAttribute(&st.sms, cudaDevAttrMultiProcessorCount, dev),
                                      "cudaDeviceGetAttribute"))
            return rc;
        st.ready = true;
    }
    *out = st;
    return VDIT_OK;
}

// One launch over `n_tok` consecutive tokens of the chunk (chunk-local first token tok0) whose K
// and V rows go to consecutive cache rows starting at cache_row0.
int launch_part(const vdit_geom* g, const vdit::RopeTables& tabs, const uint8_t* x, const void* w,
                int d_model, int start_frame, int tok0, int n_tok, uint8_t* q, void* k_cache, void* v_cache,
                long long cap_tok, long long cache_row0, const QkvDeviceState& ds, cudaStream_t st) {
    const int hd = g->heads * g->head_dim, d = g->head_dim;
    CUtensorMap mx, mw, mq, mk, mv;
    {
        cuuint64_t dims[2] = {(cuuint64_t)d_model, (cuuint64_t)n_tok};
        cuuint64_t str[1] = {(cuuint64_t)d_model * 2};
        cuuint32_t box[2] = {64, kBM};
        if (int rc = encode(&mx, x + (size_t)tok0 * d_model * 2, 2, dims, str, box)) return rc;
    }
    {
        cuuint64_t dims[2] = {(cuuint64_t)d_model, (cuuint64_t)3 * hd};
        cuuint64_t str[1] = {(cuuint64_t)d_model * 2};
        cuuint32_t box[2] = {64, kBN};
        if (int rc = encode(&mw, w, 2, dims, str, box)) return rc;
    }
    {
        cuuint64_t dims[2] = {(cuuint64_t)hd, (cuuint64_t)n_tok};
        cuuint64_t str[1] = {(cuuint64_t)hd * 2};
        cuuint32_t box[2] = {64, kBM};
        if (int rc = encode(&mq, q + (size_t)tok0 * hd * 2, 2, dims, str, box)) return rc;
    }
    for (int which = 0; which < 2; ++which) {
        cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)n_tok, (cuuint64_t)g->heads};
        cuuint64_t str[2] = {(cuuint64_t)d * 2, (cuuint64_t)cap_tok * d * 2};
        cuuint32_t box[3] = {64, kBM, 1};
        uint8_t* base = static_cast<uint8_t*>(which ? v_cache : k_cache) + (size_t)cache_row0 * d * 2;
        if (int rc = encode(which ? &mv : &mk, base, 3, dims, str, box)) return rc;
    }
    GemmArgs a{};
    a.m = n_tok;
    a.k = d_model;
    a.n_tiles_m = (n_tok + kBM - 1) / kBM;
    a.n_tiles_n = 3 * hd / kBN;
    a.n_major = (long long)3 * hd > (long long)n_tok ? 1 : 0;  // W larger than X: keep X in L2
    a.hd = hd;
    a.head_dim = d;
    a.tok0 = tok0;
    a.start_frame = start_frame;
    a.grid_h = g->grid_h;
    a.grid_w = g->grid_w;
    a.tt = static_cast<const float2*>(tabs.t);
    a.th = static_cast<const float2*>(tabs.h);
    a.tw = static_cast<const float2*>(tabs.w);
    a.bt2 = g->band_t / 2;
    a.bh2 = g->band_h / 2;
    a.bw2 = g->band_w / 2;
    a.status = ds.status;
    const int tiles = a.n_tiles_m * a.n_tiles_n;
    const int grid = std::min(tiles, ds.sms);
    qkv_rope_kernel<<<grid, kGThreads, kGSmemBytes, st>>>(mx, mw, mq, mk, mv, a);
    return vdit::cuda_check(cudaGetLastError(), "qkv_rope kernel launch");
}

}  // namespace

namespace vdit {
// Reads and clears this file's device status word (VDIT_OK or VDIT_ERR_TIMEOUT).
int qkv_status_take(int* out) {
    int zero = 0, v = 0;
    if (int rc = cuda_check(cudaMemcpyFromSymbol(&v, g_qkv_status, sizeof(int)), "read status")) return rc;
    if (int rc = cuda_check(cudaMemcpyToSymbol(g_qkv_status, &zero, sizeof(int)), "clear status")) return rc;
    *out = v;
    return VDIT_OK;
}
}  // namespace vdit

extern "C" int vdit_qkv_rope(const vdit_geom* g, const void* x, const void* w, int d_model, int start_frame,
                             int n_frames, void* q, void* k_cache, void* v_cache, int capacity_frames,
                             void* stream) {
    using vdit::fail;
    if (int rc = vdit::check_geom(g)) return rc;
    if (!x || !w || !q || !k_cache || !v_cache) return fail(VDIT_ERR_INVALID_ARG, "NULL pointer");
    auto al = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
    if (!al(x) || !al(w) || !al(q) || !al(k_cache) || !al(v_cache))
        return fail(VDIT_ERR_MISALIGNED, "tensor not 16-byte aligned");
    const long long hd = (long long)g->heads * g->head_dim;
    if (hd % kBN != 0) return fail(VDIT_ERR_UNSUPPORTED, "heads * head_dim must be a multiple of 256");
    if (d_model < 8 || d_model % 8 != 0) return fail(VDIT_ERR_INVALID_ARG, "d_model must be a positive multiple of 8");
    if (capacity_frames < 1 || n_frames < 1 || n_frames > capacity_frames)
        return fail(VDIT_ERR_INVALID_ARG, "need 1 <= n_frames <= capacity_frames");
    if (start_frame < 0 || start_frame + n_frames - 1 > VDIT_MAX_FRAME)
        return fail(VDIT_ERR_INVALID_ARG, "frames outside [0, VDIT_MAX_FRAME]");
    const long long ft = (long long)g->grid_h * g->grid_w;
    if (ft * n_frames > (1 << 30)) return fail(VDIT_ERR_UNSUPPORTED, "chunk too large");
    vdit::RopeTables tabs;
    if (int rc = vdit::get_rope_tables(g, &tabs)) return rc;
    int dev = 0;
    if (int rc = vdit::cuda_check(cudaGetDevice(&dev), "cudaGetDevice")) return rc;
    QkvDeviceState ds;
    if (int rc = qkv_device_state(dev, &ds)) return rc;
    // frames of the chunk go to slots (frame mod capacity): one launch per run of consecutive
    // slots (two when the chunk wraps around the end of the ring)
    const long long cap_tok = ft * capacity_frames;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int f = 0;
    while (f < n_frames) {
        const int slot = (start_frame + f) % capacity_frames;
        const int run = std::min(n_frames - f, capacity_frames - slot);
        if (int rc = launch_part(g, tabs, static_cast<const uint8_t*>(x), w, d_model, start_frame, (int)(f * ft),
                                 (int)(run * ft), static_cast<uint8_t*>(q), k_cache, v_cache, cap_tok,
                                 (long long)slot * ft, ds, st))
            return rc;
        f += run;
    }
    return VDIT_OK;
}
