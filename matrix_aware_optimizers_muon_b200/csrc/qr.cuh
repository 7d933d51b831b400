// The SOAP basis refresh Q <- qr(F Q): one power step and the QR of its
// result, for a bucket of q factors of equal side k (padded to kp, a
// multiple of 128, with the identity in the padded block).
//
// Arithmetic: every product runs on the tensor cores with each fp32 operand
// held as two fp16 planes, x * 2^e = h + l (h = fp16(x 2^e), l = fp16(x 2^e
// - h)), and the three plane products l h' + h l' + h h' accumulated in fp32
// (the small terms first).  With a power-of-two scale 2^e that puts the
// largest entry near 2^12..2^14, the planes carry 22 bits of each value, so
// a product is as accurate as an fp32 one.
//
// QR: CholeskyQR passes, as many as the conditioning needs.  A pass
// normalises Y's columns (the Q of Y D is Y's Q for a positive diagonal D),
// forms the Gram C = Y^T Y, factors C = L L^T by a left-looking blocked
// Cholesky with 128-wide diagonal blocks, and solves Q = Y L^{-T}.  Y and C
// are stacked as [C; Y] (2 kp rows) and the planes of L and Q as [L; Q], so
// that for block column j ONE product updates both the Cholesky panel and
// the solve:  [C; Y][128 j :, j] -= [L; Q][128 j :, < j] L[j, < j]^T.
// Then the diagonal block is factored (and inverted) by one CTA per matrix,
// and a row-block kernel multiplies the panel below it by the inverse,
// giving L's next panel and Q's block column j.
//
// Pass control, per matrix, on the device (no host synchronisation):
//   - a pass whose Gram is within tau_done of the identity (max entry) marks
//     the basis done: Y is Q and the matrix skips every later kernel;
//   - the first attempt is plain, with a pivot floor of 1e-4 (of the unit
//     diagonal): below it the factor of an ill-conditioned Gram would be
//     inaccurate, so the attempt is abandoned for that matrix and the next
//     pass is shifted (the block columns already solved stay: Y times an
//     upper-triangular matrix with a positive diagonal has Y's Q);
//   - CholeskyQR only rescales and combines Y's columns, so columns that are
//     exactly dependent (a rank-deficient factor) would stay dependent: the
//     pass after a failed attempt perturbs the normalised columns by a
//     seeded pseudo-random 1e-6 of their norm (the precision of the fp16
//     planes), which a Householder QR's completion from rounding residue
//     stands in for;
//   - a shifted pass factors C + s I with s = 1e-5 ||C||_F * mult (shifted
//     CholeskyQR: the result is still Y's Q, better conditioned); it is
//     repeated while its smallest pivot stays below 10 s, and mult grows
//     tenfold when even the shifted factorisation fails;
//   - matrices not done after the last pass get their flag set and keep
//     their previous basis.
#pragma once

#include <cuda_fp16.h>
#include <cstdint>

#include "soap_kernels.cuh"

namespace mo {

constexpr int QR_MAX_PASSES = 16;
constexpr int QR_CHECK_BLOCKS = 64;    // partial sums per matrix for the Gram check
constexpr float QR_TAU_DONE = 5e-5f;
constexpr float QR_PLAIN_FLOOR = 1e-4f;
constexpr float QR_SHIFT_REL = 1e-5f;
constexpr float QR_NOISE = 1e-6f;              // relative perturbation after a failed attempt
constexpr float QR_PLANE_SCALE = 4096.f;       // 2^12: planes of L and Q (|L|, |Q| <= 16)
constexpr float QR_Y_SCALE = 16384.f;          // 2^14: planes of the normalised Y and of Q_old (|x| <= 1)

// Per-matrix control state of one bucket (device arrays of q entries).
struct QrCtl {
  int* done;            // the basis passed the orthonormality check
  int* skip;            // this pass: the matrix takes no part (done, or its factorisation failed)
  int* fail;            // this pass: a pivot fell to or below the floor
  int* mode;            // this pass: 1 shifted, 0 plain, -1 no attempt
  int* next_shift;      // the next attempt runs shifted
  float* mult;          // multiplier of the shift
  float* floor;         // this pass: pivot floor
  float* shift;         // this pass: shift added to the Gram's diagonal
  unsigned* minpiv;     // this pass: smallest pivot (bits of a positive float)
  unsigned* dev;        // this pass: max |C - I| (bits of a non-negative float; NaN above all)
  float* part;          // [q][QR_CHECK_BLOCKS] partial sums of C_ij^2
  float* fscale;        // power step: scale 2^e of the factor's planes
  float* fiscale;       // and its inverse
  int* pass_done;       // [QR_MAX_PASSES]: matrices done after pass p's decision
  int* npass;           // passes run so far (the pass loop recorded as a graph reads it)
};

// Bytes of the control arrays for q matrices (1024-byte aligned pieces).
size_t qr_ctl_bytes(int q);
QrCtl qr_ctl_at(char* base, int q);

// done = 0, mode = -1, next_shift = 0, mult = 1, dev = 0
void launch_qr_init(const QrCtl& c, int q, cudaStream_t s);

// fscale[b] = 2^(13 - ceil(log2 m_b)), fiscale = 1 / fscale, with m_b the
// largest diagonal entry of the k x k factor F[b] (plus delta[b] when given):
// the largest entry of a positive semi-definite matrix sits on its diagonal.
struct FactorScaleArgs {
  int count, k;
  const float* F[SOAP_MAXB];
  const float* delta;               // optional damping per matrix
};
void launch_factor_scale(const FactorScaleArgs& a, const QrCtl& c, cudaStream_t s);

// Two fp16 planes of fp32 matrices, 8 columns per thread.  Value of element
// (r, c) of matrix b: src[b][r * lds + c] (+ diag_add[b] on the diagonal),
// times col_scale[b * cols_pad + c] when given (a zero there replaces the
// column by the unit vector e_c), for r < rows_valid and c < cols_valid;
// elsewhere 0, or 1 on the diagonal with pad_identity.  Planes of x * scale
// (scale = mscale[b], or cscale) go to dst + p * plane_stride + b *
// mat_stride + r * ldd + c; write_back (optional) receives the fp32 value.
// cols_valid, cols_pad, lds, ldd and ldw are multiples of 8.
struct Split16Args {
  int count, rows_valid, cols_valid, rows_pad, cols_pad;
  const float* src[SOAP_MAXB];
  long long lds;
  const float* diag_add = nullptr;
  const float* col_scale = nullptr;
  const float* mscale = nullptr;
  float cscale = 1.f;
  float* write_back = nullptr;
  long long ldw = 0, wb_stride = 0;
  __half* dst;
  long long ldd, mat_stride, plane_stride;
  int pad_identity = 0;
  const int* skip = nullptr;
  // optional: matrices with noise_on[b] != 0 get, after the column scale, a
  // pseudo-random perturbation of noise_amp / sqrt(cols_pad) per entry
  // (uniform in [-1, 1), a hash of b, r, c and noise_seed)
  const int* noise_on = nullptr;
  float noise_amp = 0.f;
  unsigned noise_seed = 0u;
  const int* gate = nullptr;          // launch gate (see launch_qr_control)
  int gate_n = 0;
  const int* seed_dev = nullptr;      // optional: the noise seed read from device memory
};
// The padded diagonal (pad_identity) is written as min(scale, 2^14) in the
// planes, whatever the scale, so that it never overflows fp16; write_back
// receives 1 there.
void launch_split16(const Split16Args& a, cudaStream_t s);

// inv_d[b][c] = 1 / ||Y[b][:, c]|| (0 for a zero column, NaN for an
// infinite norm) over the first `rows` rows; skips matrices with skip[b].
void launch_colnorm2(const float* Y, long long ld, long long mat_stride, int count, int rows, int cols,
                     float* inv_d, const int* skip, const int* gate, int gate_n, cudaStream_t s);

// Launch gate (optional, device): the launch does nothing when *gate >=
// gate_n (every matrix of the refresh already done).  The refresh kernels
// launch with programmatic stream serialization: each waits for its
// predecessor before its first global access, so a gated-off pass costs a
// few microseconds per launch.
// pass_done[pass] counts the matrices done after this pass's decision: the
// gate of this pass's block steps and of the next pass's launches.
//
// The Gram check and the pass decision: max |C - I| and sum C^2 of each kp x
// kp Gram (fixed-order partial sums; the check is gated by `gate`), then per
// matrix the decision above, with the shift added to C's diagonal.
// `pass_dev` (optional) replaces `pass` by a device word.
void launch_qr_control(const float* C, long long ld, long long mat_stride, int q, int kp, const QrCtl& c,
                       int pass, const int* pass_dev, const int* gate, cudaStream_t s);

// End of one pass of the pass loop recorded as a graph (a conditional while
// node): npass += 1, and the loop goes on while a matrix is not done and
// fewer than QR_MAX_PASSES passes have run.
void launch_qr_loop(const QrCtl& c, int q, cudaGraphConditionalHandle h, cudaStream_t s);

// Diagonal block j of each matrix's Cholesky factor: C[b] + (128 j)(ld + 1)
// holds the 128 x 128 Schur complement block; factor it with the matrix's
// pivot floor, record the smallest pivot, and write the inverse of the
// lower factor, transposed (an upper-triangular 128 x 128 matrix), to
// Dinv[b].  A pivot at or below the floor sets fail[b] and skip[b].
void launch_qr_chol(const float* C, long long ld, long long mat_stride, int q, int j, float* Dinv,
                    const QrCtl& c, const int* gate, const int* gate_idx, cudaStream_t s);

// Rows [r0, r1) of each matrix's stacked [C; Y] (row stride ld), block
// column j: x = row * Dinv^T (128 wide).  Its fp16 planes (scale
// QR_PLANE_SCALE) go to the same place in the stacked planes [L; Q]; rows
// >= f32_from also keep x in fp32 (Q's block column).
struct PanelArgs {
  int q, j, r0, r1, f32_from;
  float* CY; long long ld, mat_stride;
  const float* Dinv;
  __half* LQ; long long plane_stride;     // planes: same ld and mat_stride as CY
  const int* skip;
  const int* gate = nullptr;              // launch gate: nothing when gate[gate_idx ? *gate_idx : 0] >= q
  const int* gate_idx = nullptr;
};
void launch_qr_panel(const PanelArgs& a, cudaStream_t s);

// After the last pass: flag[b] = 1 for every matrix whose basis is not done,
// and its Y (kp x kp, row stride ld) reset to its previous basis Qold[b]
// (k x k, padded with the identity), so that a failed refresh keeps the old
// basis instead of a non-orthonormal iterate.
void launch_qr_finish(const QrCtl& c, const FlagTable& flags, int q, float* Y, long long ld,
                      long long mat_stride, int k, int kp, const float* const* Qold, cudaStream_t s);

}  // namespace mo
