// Internal helpers shared by the libvdit translation units (not part of the C ABI).
#pragma once

#include <cstdint>
#include <string>
#include <vector>

#include "vdit.h"

namespace vdit {

// Records msg as this thread's last error and returns code.
int fail(int code, const std::string& msg);
// Maps a cudaError_t (as int) to VDIT_ERR_CUDA with the CUDA message, or VDIT_OK.
int cuda_check(int err, const char* what);

// Validates a geometry (bands, head_dim, grid); returns VDIT_OK or an error already recorded.
int check_geom(const vdit_geom* g);

// Device RoPE tables for one band set on the current device: float2 (cos, sin) rows
//   t: (VDIT_MAX_FRAME + 1) x band_t/2, h: VDIT_MAX_GRID x band_h/2, w: VDIT_MAX_GRID x band_w/2,
// built once in fp64 on the host ([CRoPE] 2.C: precomputed contiguous tables, no per-call host
// work). Returned pointers stay valid until process exit.
struct RopeTables {
    const void* t;  // float2*
    const void* h;
    const void* w;
};
int get_rope_tables(const vdit_geom* g, RopeTables* out);
// Same tables, lookup only (never allocates); an error if they were never built on this device.
int find_rope_tables(const vdit_geom* g, RopeTables* out);

// Reads and clears the device status word of the fused QKV projection kernel.
int qkv_status_take(int* out);

// Size of the attention module's fixed no-allocation scratch buffer, and the number of key-piece
// partial results (256 query rows x (head_dim + 1) fp32 each: normalised O and log2-sum-exp) that
// it holds. The schedule never uses more slots than this, so every plan fits the buffer.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB
constexpr int max_partial_slots(int head_dim) {
    return (int)(kNoAllocScratchBytes / (256u * 4u * (size_t)(head_dim + 1)));
}

// One-time set-up of the attention kernels on device dev (current): shared-memory opt-in of every
// kernel instance, device addresses of the status word and of the no-allocation scratch buffer.
int attn_prepare_device(int dev);

}  // namespace vdit

// Plan object (host schedule + optional device copy).
struct vdit_plan {
    vdit_geom g;
    vdit_mask m;
    int q_start, q_frames, cap_frames, kv_first, kv_last;
    int q_tokens, kv_tokens, n_qt, n_kt;
    int n_full;
    int dt_max;  // largest |t_q - t_k| over query frames x held key frames
    long long kept_pairs;
    std::vector<int> row_ptr, col_idx;
    std::vector<unsigned char> full;
    std::vector<int> slot_frame;  // global frame held by each frame slot, -1 if empty
    std::vector<int> radius;      // per dt in [0, dt_max]: largest kept Chebyshev distance
    // Blocks of two consecutive q-tiles (2b, 2b+1), the unit one attention CTA works on: the
    // union of the two tiles' work lists (aligned entries merged by key row, ascending; then the
    // single-patch entries, each for one q-tile), with per entry
    //   bit0: listed for q-tile 2b, bit1: full for 2b, bit2: listed for 2b+1, bit3: full for 2b+1.
    int n_qb = 0;
    std::vector<int> u_row_ptr, u_col;
    std::vector<unsigned char> u_flags;
    std::vector<int> unit_order;  // q-blocks by descending union-list length (longest first)
    // keep masks of the partial tiles: mask_of[i] = block of CSR entry i (-1: full tile); block b
    // = masks[512 b ..): 128 rows x 4 words, bit k of row r = key k of the tile kept for query r.
    // u_mask[2 e + x] = block in kmasks of union entry e for q-tile 2b + x (-1: not listed or full)
    std::vector<int> mask_of;
    std::vector<uint32_t> masks;
    std::vector<int> u_mask;
    // The kernel's work list, per q-tile: entries (first key row, keep-mask block or -1 for a full
    // tile) in kmasks. It holds the listed tiles above, except that for frames whose radial
    // window is a single patch (radius 0) the kept "same patch" pairs of a q-tile are taken out of
    // the aligned tiles into one entry at an unaligned key row: query row r of the q-tile meets
    // key row w_key + r, the same patch dt frames away (when that moves work off the tensor path).
    // The union lists u_* are built from this list (u_col holds first key rows).
    std::vector<int> w_row_ptr, w_key, w_mask;
    std::vector<int> w_aligned;   // per q-tile: its first w_aligned[qt] entries are aligned tiles
    std::vector<uint32_t> kmasks;
    int n_diag = 0;               // entries of the single-patch kind
    // CTA schedule of the attention kernel, fixed at upload from the device's SM count:
    //   cta[5 i ..]: q-block, head, first union entry of the piece (within the unit), entries,
    //                partial slot (-1: the unit runs whole and writes O itself);
    //   merge[4 j ..]: a unit cut into pieces: q-block, head, first slot, pieces (slots
    //                  first .. first + pieces - 1, merged by the second kernel).
    std::vector<int> cta, merge;
    int n_slots = 0;
    int n_split = 1;  // most pieces of one unit
    // device copy
    int device = -1;
    void* d_buf = nullptr;
    const int* d_u_row_ptr = nullptr;
    const int* d_u_col = nullptr;
    const unsigned char* d_u_flags = nullptr;
    const int* d_cta = nullptr;        // int4 per CTA: q-block, head, first entry, entries
    const int* d_cta_slot = nullptr;   // per CTA: partial slot or -1
    const int* d_merge = nullptr;      // int4 per cut unit: q-block, head, first slot, pieces
    const uint32_t* d_masks = nullptr;
    const int* d_u_mask = nullptr;
    float* d_ws_o = nullptr;    // [slots][256 query rows][head_dim] normalised partial O
    float* d_ws_lse = nullptr;  // [slots][256 query rows] partial log2-sum-exp
    size_t ws_bytes = 0;
};
