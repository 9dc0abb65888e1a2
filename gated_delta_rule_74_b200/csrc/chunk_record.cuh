// Layout of the chunk record the prep kernel writes for one (head, chunk): the
// chunk-only operands of the chunked form (device code shared by the split prefill
// and the chunked backward; not part of the C ABI).
//
// Images.  Every bf16 / f16 image below is a matrix with 64 columns stored as
// 128-byte rows whose 16-byte chunks (8 columns each) are XOR-swizzled with
// (row % 8): element (row, col) sits at byte
//     row * 128 + (((col / 8) ^ (row % 8)) * 16) + (col % 8) * 2.
// Stacked 64-column panels of an image with R rows follow each other R * 128
// bytes apart.  The same bytes are the tensor cores' 128-byte-swizzled operand
// tile and a bank-conflict-free ldmatrix source.
#pragma once

#include <stdint.h>

namespace kda {
namespace rec {

// [Qbar^T | W^T]: rows = key channel c (128), columns = token; Qbar^T at +0,
// W^T at +16384 (bf16)
constexpr uint32_t QW = 0;
// [Kend^T ; Aqk]: Kend^T rows = key channel, columns = token (16 KB); then Aqk,
// rows = token r, columns = token i (8 KB).  f16 in the prefill's records, bf16 in
// the backward's.
constexpr uint32_t KA = 32768;
constexpr uint32_t AQK = KA + 16384;
// U^T: rows = value channel j, columns = token (f16 prefill / bf16 backward)
constexpr uint32_t U = 57344;
// exp(Gamma_last) per key channel, fp32 [128]
constexpr uint32_t DECAY = 73728;
constexpr uint32_t BYTES = 74240;           // prefill record
// backward record only: T = (I + diag(beta) A)^-1 as a bf16 image [64 r][64 i] (8 KB, the
// layout above), then A (unscaled, strictly lower) in fp32 [64][64] row-major
constexpr uint32_t TMAT = 74240;
constexpr uint32_t AMAT = TMAT + 8192;
constexpr uint32_t BYTES_BWD = AMAT + 16384;  // 98,816

}  // namespace rec
}  // namespace kda
