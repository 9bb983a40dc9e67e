// A 16-level code book: level j of code j, in increasing order over [-1, 1] (two equal
// neighbours allowed, as the two zeros of E2M1).  Kernels take it by value in their
// parameters, so that the constant-index reads of the unrolled table builds are plain
// parameter operands.
#pragma once

namespace qnf4 {

struct Codebook {
  float q[16];
};

}  // namespace qnf4
