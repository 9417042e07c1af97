// Internal declarations shared by the host library and the kernel launchers.
#pragma once

#include <cstdint>
#include <string>
#include <vector>

#include "../../include/mosaicq.h"

namespace mq {

constexpr int kGroup = 128;
constexpr int kBlockRows = 16, kBlockCols = 64;  // residual blocks (block mode)

// Thread-local "last error" text behind mq_last_error().
void set_error(const std::string &msg);
mq_status fail(mq_status s, const std::string &msg);

// ---- host decomposition and packing (host_pack.cpp; no CUDA calls) ----

// fp64 -> fp16 bits, one round-to-nearest-even step; overflow gives +-inf.
uint16_t f64_to_f16_bits(double x);
double f16_bits_to_f64(uint16_t h);

// Unpacked decomposition held by the host while packing.
struct HostDecomp {
    int64_t N = 0, K = 0;
    std::vector<uint8_t> q;        // [N][K]
    std::vector<uint16_t> s, z;    // [N][G] fp16 bits
    std::vector<int64_t> row_ptr;  // [N+1]
    std::vector<int32_t> col;      // [nnz]
    std::vector<int8_t> qr;        // [nnz]
    std::vector<uint16_t> sr;      // [N] fp16 bits
};

// Packed layout in host memory; sz rows are padded to a multiple of 4 words
// (16 bytes) so the device copy can be read by TMA.
struct HostPacked {
    int64_t N = 0, K = 0, G = 0, Gp = 0, nnz = 0;
    std::vector<uint32_t> qweight;  // [N][K/8]
    std::vector<uint32_t> sz;       // [N][Gp], zero padding
    std::vector<int32_t> row_ptr;   // [N+1]
    std::vector<uint16_t> col;      // [nnz]
    std::vector<uint8_t> val;       // [(nnz+1)/2]
    std::vector<uint16_t> rscale;   // [N]
};

// Block tiles of a residual made of whole 16 x 64 blocks on the block grid
// (the block allocation): per block-row offsets, column-block indices, and
// per block 16 rows x 8 words of offset-binary codes q_r + 8 in the base
// codes' nibble interleave. `map` (device helper, not part of the packed
// form) has one bit per column-block for every block-row, words of 32.
struct HostBlocks {
    int64_t nblk = 0, map_words = 0;
    std::vector<int32_t> ptr;   // [N/16 + 1]
    std::vector<uint16_t> col;  // [nblk]
    std::vector<uint32_t> q;    // [nblk][16][8]
    std::vector<uint32_t> map;  // [N/16][map_words]
};

// Builds the tiles when the packed residual is block-structured: N % 16 == 0,
// K % 64 == 0, and each row of a block-row holds exactly the columns of the
// same aligned 64-column runs. Returns false (and leaves `b` empty)
// otherwise, or when there is no residual.
bool block_tiles_host(const HostPacked &p, HostBlocks &b);

mq_status check_shape(int64_t N, int64_t K, const mq_pack_opts *opts);
int64_t residual_count(int64_t K, double rho);
mq_status decompose_host(const float *W, int64_t N, int64_t K, const mq_pack_opts &opts,
                         HostDecomp &d);
int64_t residual_blocks_selected(int64_t N, int64_t K, double fraction);
mq_status validate_decomp(const mq_decomp *d);
void pack_host(const mq_decomp &d, HostPacked &p);
mq_decomp view_of(const HostDecomp &d);

}  // namespace mq
