// qfp4_internal.h - declarations shared by the library's translation units
// (not part of the public ABI; include/qfp4.h is).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace qfp4 {

constexpr int kNvfp4 = 0, kMxfp4 = 1;
constexpr int kRtn = 0, kSr = 1, kQuartet2 = 2;
constexpr int kTagElement = 0, kTagScale = 1, kTagSign = 2;

// Upper bound on the number of per-CTA amax partials (the workspace holds them).
constexpr int kMaxAmaxPartials = 1024;

struct QuantParams {
    const uint16_t* x;  // bf16 input, R x C, row stride ld
    int64_t R, C, ld;
    int64_t rows, k;  // quantized orientation
    uint8_t* codes;
    uint8_t* scales;
    float* tensor_scale;
    int64_t kb4;                  // scale columns padded to a multiple of 4
    const float* amax_partials;   // NVFP4: partial maxima from the amax pass
    int n_partials;
    const float* amax_in;         // NVFP4: caller-provided amax (overrides partials)
    float* amax_out;              // amax pass: partial maxima written here
    uint32_t signs;               // random Hadamard sign bits (0 for deterministic / none)
    // Row-and-column amax pass (column kernel): the row orientation's sign bits
    // and partial maxima.
    uint32_t signs_row;
    float* amax_out_row;
    uint64_t sr_seed;
    uint32_t sr_tag_elem;         // kTagElement | stream << 4
    uint32_t sr_tag_scale;        // kTagScale | stream << 4
    uint32_t mx_round_up;         // MXFP4: 1 = the smallest E with amax_b <= 6 * 2^E (no clipping)
    // Dual quantization (the column kernel over 64-row bands also quantizes
    // x along its rows): the row orientation's outputs, tensor amax and
    // randomness; its sign bits are signs_row.
    uint8_t* codes_row;
    uint8_t* scales_row;
    float* tensor_scale_row;
    const float* amax_in_row;
    int64_t kb4_row;
    uint64_t sr_seed_row;
    uint32_t sr_tag_elem_row;
    uint32_t sr_tag_scale_row;
    // Fused amax and quantization (one cooperative launch): the grid barrier's
    // arrival counter, zeroed before the launch; the partials go to amax_out
    // and are read back through amax_partials.
    uint32_t* grid_counter;
};

// Launchers (quant.cu). Return cudaSuccess or the launch error.
// `tmap` is the TMA view of x: 2-D (row mode) or the 5-D column view.
cudaError_t launch_amax(const QuantParams& p, int axis, int nh, const CUtensorMap* tmap, int n_partials,
                        cudaStream_t s);
// axis: 0 row, 1 column (5-D group view), 2 column over 64-row bands (the
// 4-D band view; quantized axis a multiple of 64).
cudaError_t launch_quant(const QuantParams& p, int fmt, int rnd, int nh, int axis, const CUtensorMap* tmap,
                         cudaStream_t s);
// NVFP4 amax and quantization in one cooperative launch (a first pass takes the
// rotated amax, a grid barrier, then the quantizing pass re-reads the tiles,
// from L2 for a tensor that fits there): rnd RTN or Quartet II, nh 0 or 16,
// axis 0 (row) or 2 (64-row bands). p.amax_out == p.amax_partials (room for
// 2 x SM count partials) and p.grid_counter (zeroed) are set by the caller.
cudaError_t launch_quant_fused(const QuantParams& p, int rnd, int nh, int axis, const CUtensorMap* tmap,
                               cudaStream_t s);
// Dual quantization of x (R x C, R a multiple of 64; tmap: the 64-row band
// view): p describes the column orientation, p.*_row the row orientation.
// nh: the column orientation's Hadamard size; nh_row: 0 or nh.
cudaError_t launch_quant_dual(const QuantParams& p, int fmt, int rnd, int nh, int nh_row, const CUtensorMap* tmap,
                              cudaStream_t s);
// One pass of the column kernel (tmap: its 5-D view, group 16) that writes the
// column orientation's partial maxima to p.amax_out and the row orientation's
// to p.amax_out_row (n_partials each). nh: 0 or 16.
cudaError_t launch_amax_rowcol(const QuantParams& p, int nh, const CUtensorMap* tmap, int n_partials, cudaStream_t s);
// The same over 64-row bands (R a multiple of 64; tmap: the 4-D band view),
// both orientations as two packed pairs of 16-element groups per thread.
cudaError_t launch_amax_rowcol64(const QuantParams& p, int nh, const CUtensorMap* tmap, int n_partials,
                                 cudaStream_t s);
// Tiles the band amax pass walks (rows, k of the column orientation).
int64_t amax_rowcol64_tiles(int64_t rows, int64_t k);
cudaError_t launch_reduce_max(const float* in, int n, float* out, cudaStream_t s);
// Column-mode geometry: group G = max(block, n_h), tile = 4G rows x 128 columns.
int col_group(int fmt_or_amax_block, int nh);
// Number of tiles a quantizer (or amax) pass walks (G: the column-mode group).
int64_t quant_tiles(int axis, int64_t rows, int64_t k, int G);
// SM count of the current device (sizes the persistent grids).
void set_sm_count(int sms);

struct GemmParams {
    const uint8_t* sfa;
    const uint8_t* sfb;
    const float* ga;
    const float* gb;
    void* D;
    int64_t ldd;
    int out_f32;
    int accumulate;  // fp32 output only: D += result (one fp32 add per element)
    // bf16 output only, pair kernel: the output also quantized to MXFP4 along
    // N (round to nearest, Hadamard of the kernel's NHQ with these sign bits),
    // codes [M][N/2] and scales in the atom layout (q_kb4 scale columns)
    uint8_t* q_codes;
    uint8_t* q_scales;
    int64_t q_kb4;
    uint32_t q_signs;
    // bf16 output only, pair kernel: the NVFP4 tensor amax of the output along
    // its rows after the next layer's rotation (the kernel's AMX size, these
    // sign bits): one partial maximum per CTA into amax_partials[blockIdx.x]
    float* amax_partials;
    uint32_t amax_signs;
    int M, N, K;
    int atoms_k;  // scale atoms per 128-row block along k: ceil(K / block / 4)
};

// gemm_sm100.cu
cudaError_t launch_gemm(const GemmParams& p, int fmt, const CUtensorMap* tmapA, const CUtensorMap* tmapB,
                        cudaStream_t s, int sms);
// 2-SM (CTA pair) variant; tmapSFA / tmapSFB are 3-D views of the scale
// buffers, tmapD a 2-D view of D for TMA stores (see make_scale_tmap and
// make_out_tmap in qfp4_api.cu).
// nhq: -1 (no quantized output) or the Hadamard size (0, 16, 32) of the
// MXFP4 output quantization (p.q_codes etc.).
// amx: -1 (no amax of the output) or the Hadamard size (0, 16, 32) of the
// output's tensor amax (p.amax_partials; *n_partials receives their count).
cudaError_t launch_gemm_pair(const GemmParams& p, int fmt, const CUtensorMap* tmapA, const CUtensorMap* tmapB,
                             const CUtensorMap* tmapSFA, const CUtensorMap* tmapSFB, const CUtensorMap* tmapD,
                             cudaStream_t s, int sms, int nhq = -1, int amx = -1, int* n_partials = nullptr);
constexpr int kGemmBM = 128, kGemmBN = 256, kGemmBK = 256;

void count_launch();

}  // namespace qfp4
