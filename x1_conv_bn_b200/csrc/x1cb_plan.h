// Launch plan of the fused implicit-GEMM convolution: geometry, tiling,
// shared-memory carve-up.  Computed on the host, passed to the kernel by value.
#pragma once
#include <cstdint>

namespace x1cb {

constexpr int kEpiWarp0 = 4;        // warps 0-3: producers, MMA issuer, store
constexpr int kEpiWarps = 16;       // 4 per TMEM lane quarter
constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);
constexpr int kAIssuers = 4;            // lanes of the producer warp issuing activation copies
constexpr unsigned kAIssuerMask = (1u << kAIssuers) - 1;
static_assert(kEpiWarp0 % 4 == 0 && kEpiWarps % 4 == 0, "roles must be whole warpgroups");
constexpr int kTileRows = 128;      // MMA M
constexpr int kKBlock = 32;         // int8 channels per K block (one MMA K step)
constexpr int kASlotBytes = kTileRows * kKBlock;  // 4 KB per A ring slot
constexpr int kRChunks = 4;         // 32-channel chunks per residual stage
constexpr int kRSlotBytes = kRChunks * kTileRows * 32;  // 16 KB
constexpr int kTmemCols = 512;
constexpr int kSmemLimit = 232448;  // 227 KB opt-in per block on sm_100

// Status bits of the device status word.
constexpr unsigned kDevTimeoutProducer = 1u;
constexpr unsigned kDevTimeoutMma = 2u;
constexpr unsigned kDevTimeoutEpilogue = 4u;
constexpr unsigned kDevDrainFailed = 8u;

struct ConvPlan {
    // problem
    int B, H, W, Ic, Oc, R, pad;  // R, pad: filter height and its padding
    int Rw, padw;                  // filter width and its padding (R, pad unless folded)
    int C1, O1;       // Ic/32, Oc/32
    int Wp, Hp;       // output spatial dims seen by the tensor maps (1x1: H*W and 1)
    // Convolution stride and the input image the activation map covers
    // (Wpi, Hpi: the input's dims as the map sees them; H*W and 1 for a
    // stride-1 1x1).  Output pixel (h, w) reads input rows h*stride + dr - pad.
    int stride, Hin, Win, Wpi, Hpi;
    int stride_w;  // column stride (the folded stem: 1, its fold applied the 2)
    // Optional second activation source whose K blocks follow the first's in
    // the same accumulator (the projection shortcut of a downsampling block):
    // a 1x1 at stride `stride2` over a Hin2 x Win2 image of C1b channel blocks.
    // kb_a = R*R*C1 blocks come from the first source, C1b from the second.
    int C1b, kb_a, stride2, Hin2, Win2;
    int has_res;
    int S;
    int m_r;
    // M tile: tw x th pixels of tg images (rows = tw*th*tg <= 128)
    int tw, th, tg, rows;
    int nTw, nTh, nTg;
    int num_m_tiles;
    // N split: each CTA keeps NC output channels' weights resident
    int NC, n_groups, nmma, n_subs;
    int O2;        // output channels per weight block: 128, or Oc for a 64-channel layer
    int stage_ch;  // 32-channel chunks per I/O stage: 4, or 2 for a 64-channel layer
    int n_slots;   // accumulator slots in TMEM (512 columns / nmma)
    // MMA issuing warps, 1 or 2.  One thread issues a tcgen05.mma only every
    // ~90 cycles, while an N <= 128 MMA takes 64 tensor cycles or less; a
    // layer without a shortcut has no shortcut loads for warp 2, so warp 2
    // can be a second MMA issuer (warp 1 takes the CTA's even tiles, warp 2
    // the odd ones; each owns half of the activation ring and the accumulator
    // slots of its tiles, n_slots even) while the store warp hands the I/O
    // stages back out.  Used where it measured faster: the folded stem.
    int n_mma_warps;
    // CTA pairs (shortcut layers whose NC = 256 weights take more than 96 KB):
    // clusters of two CTAs of one channel group share each MMA (M = 256, each
    // CTA's 128 rows), each holding half of every K block's weights; grid
    // counts CTAs (two per cluster).
    int pair;
    int kb_per_tile;  // R*R*C1
    int a_kc;         // K blocks per activation TMA box (divides C1)
    int a_slot;       // bytes per ring stage: activation part + streamed weights
    int a_part;       // bytes of the activation part of a stage (a_kc * 4 KB, or the halo tile)
    // Streamed weights (when a resident copy of NC channels does not fit):
    // every stage also carries its K blocks' weights, w_part bytes right after
    // the activation part (each K block NC rows x 32 bytes; the halo form: all
    // nine taps of the stage's channel block).  0 = weights resident.
    int wstream, w_part;
    // rings
    int a_stages, r_stages;
    // shared memory offsets from the 1024-aligned base
    int off_w, off_a, off_r, off_cc, off_cm, off_bar, off_misc;
    int smem_bytes;  // including alignment slack
    int io_wide;  // shortcut/output maps use 8-byte elements (box rows of tw*32 bytes)
    // Shortcut/output stages use the TMA's 128-byte swizzle: box rows of 128
    // bytes (4 pixels of one chunk) whose 16-byte units are permuted by the
    // row index, so the epilogue's per-pixel 32-byte accesses avoid bank
    // conflicts.  Needs tw and the stored row length to be multiples of 4.
    int io_swz;
    // Shared memory reserved for folding the bias into the MMA (0 = no room):
    // a constant 128 x 32-byte A tile at off_ba and NC x 32 bytes of per-channel
    // digit rows at off_bb.
    int fold_room, off_ba, off_bb;
    // Halo form of the 3x3 convolution: one activation slot per channel block
    // holds tg images x (th+2) rows x (tw+2) columns around the tile (no
    // swizzle, the two 16-byte K halves `a_half` bytes apart), and every
    // filter tap reads it shifted by dr*(tw+2)+ds rows.  GEMM row m of the
    // tile is pixel (g, y, x) with m = (g*(th+2) + y)*row_pitch + x.
    // halo = 2: the stride-2 3x3 over four phase planes.  halo = 3: a column
    // filter (R x 1, row stride 2, column stride 1) over a width-folded image
    // with one channel block, pooled: one slot holds the 2*th + R - 2 input
    // rows of the tile's tw = 8 columns (32-byte swizzle, one 256-byte atom
    // per input row), and tap dr reads it dr rows on with 512 bytes between
    // GEMM row groups (output row y reads input row 2y + dr).
    int halo;
    int row_pitch;  // GEMM rows per image row: tw, or tw+2 in the halo form
    int plane_m;    // GEMM rows per image of the tile: tw*th, or (th+2)*(tw+2)
    int a_half;     // halo form: bytes between the two K halves of a slot
    // Max pooling fused after the ReLU (3x3, stride 2, pad 1): tiles cover
    // pw x ph pooled pixels; their conv tile is (2pw+1) x (2ph+1) pixels from
    // conv pixel (2*pooled origin - 1), so neighbouring tiles share one conv
    // row/column.  Conv pixels outside the conv output count as 0, which never
    // wins over a ReLU output.  The pooled tile is staged in the upper half of
    // the I/O stage and stored to the pooled tensor (Hpo x Wpo).
    int pool, pw, ph, Hpo, Wpo;
    // control
    int inject;  // test hook: 1 = the MMA warp waits on a barrier nobody arrives on
    unsigned long long wait_limit_ns;
    int grid;
    unsigned long long *trace;  // timeline table (trace builds only; else null)
};

// Launch plan of the fused Conv2 -> Conv3 kernel (pairs of CTAs; see
// x1cb_chain.cu).  Conv2 is the 3x3 (pad 1, halo tiles of th rows x tg
// images, full width); Conv3 the 1x1 with the shortcut.
struct ChainPlan {
    int c3;  // 1: Conv2 -> Conv3 fused; 0: the 3x3 alone (Cout = Cm, stored like Conv3)
    // The 3x3 alone at stride 2 (stride = 2): input Hin x Win, the halo tile
    // as four phase planes of (th+1) x (W+1) pixels (see the convolution
    // kernel's stride-2 halo form).
    int stride, Hin, Win;
    int issuers;  // the 3x3 alone: MMA-issuing warps (2: even / odd pair tiles, half a ring each)
    int B, H, W, Cm, Cout, S, m_r;
    int C1, n_chunks;  // Cm/32 channel blocks, Cout/128 output chunks
    int th, tg, tw, row_pitch, plane_m, a_half, rows;
    int nTh, nTg, num_m_tiles, n_pairs;
    int a_stages, a_slot, r_stages;
    int off_w2, off_w3, off_a, off_a3, off_r, off_cm2, off_cc2, off_cm3, off_cc3, off_bar,
        off_misc;
    int smem_bytes;
    int io_swz;  // output/shortcut stages in the 128-byte swizzle (else 8-byte-element rows)
    int grid;    // CTAs (two per cluster)
    unsigned long long wait_limit_ns;
    unsigned long long *trace;  // timeline table (trace builds only; else null)
};

}  // namespace x1cb
