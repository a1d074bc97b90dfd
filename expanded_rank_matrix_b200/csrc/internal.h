// Internal interfaces between the C-ABI layer and the kernels.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace externd {

struct SeqHostArgs {
  const float* A;
  int64_t m, n, k;
  float tau;
  int iters;
  const float* w;
  uint32_t* packed_B;
  uint32_t* packed_C;
  float* D;
  double* energy;
  int64_t ntrace;
  const int64_t* trace_comp;
  uint32_t* trace_bits;
  int32_t* trace_row;
  uint8_t* trace_flags;
  int64_t* stats;
  int64_t wait_budget;
  unsigned flags;         // EXTERND_TSTAT_MEAN_ABS | EXTERND_VSTEP_NAIVE
  int sweeps;             // refinement sweeps after the greedy pass
  double* sweep_energy;   // [sweeps] out (device), may be NULL when sweeps == 0
};

struct BlockHostArgs {
  const float* A;
  int64_t m, n, k;
  float tau;
  int iters;
  const float* w;
  int block;
  uint32_t* packed_B;
  uint32_t* packed_C;
  float* D;
  double* energy;
  int64_t* stats;
  int64_t ntrace;
  const int64_t* trace_block;  // host array: traced block indices
  uint64_t* trace_uv;          // device: per traced block, V0 then U_t, V_t masks
  int32_t* trace_rows;         // device: per traced block, the start rows
  unsigned flags;              // EXTERND_TSTAT_MEAN_ABS | EXTERND_VSTEP_NAIVE
  int64_t wait_budget;         // SM cycles for the contractions' waits (0: default)
};

int seq_decompose(const SeqHostArgs& h, cudaStream_t st);
int block_decompose(const BlockHostArgs& h, cudaStream_t st);
int reconstruct(const uint32_t* pB, const uint32_t* pC, const float* D, int64_t m, int64_t n,
                int64_t k, float* out, cudaStream_t st);
int* status_word_ptr();
int ternary_apply(const uint32_t* pB, const uint32_t* pC, const float* D, int64_t m, int64_t n,
                  int64_t k, const float* X, int64_t nb, float* Y, cudaStream_t st);
// Block-ALS contractions on the tensor cores.  Vm/Vs (Um/Us) are the 64-bit
// per-entry masks of the ternary operand, Bop the same codes as bf16 B chunks
// (4 KB per 32 entries); wpad the weights zero padded to a multiple of 32.
// With a plan (and 16-byte aligned rows of R) the persistent TMA kernel runs
// and writes stream-K tile partials Xp[(t S + slot) 128 + row][bb]; otherwise
// the direct kernel writes split-K partials Xp[split][row][bb].
constexpr int kMaxSegs = 16;  // partials summed per output row, either layout
struct TcPlan {
  int T, C, G, S;  // tiles of 128 rows, chunks of 32 along K, CTAs, slots per tile
  long long U;     // T * C units
};
void tc_contract_plan(int M, int Kdim, int nsm, TcPlan* p);
bool tc_contract_tma_ok(int n);  // n % 4 == 0 and the tensor-map encoder is available
int tc_contract_rv(const float* R, int m, int n, const unsigned long long* Vm,
                   const unsigned long long* Vs, const unsigned char* Bop, const float* w,
                   const float* wpad, int bb, const TcPlan* p, int klen, int splits, float* Pp,
                   long long budget, cudaStream_t st);
int tc_contract_rtu(const float* R, int m, int n, const unsigned long long* Um,
                    const unsigned long long* Us, const unsigned char* Bop, int bb, const TcPlan* p,
                    int klen, int splits, float* Qp, long long budget, cudaStream_t st);
int block_release_graphs();
int apply_trim_pools();
int seq_decompose_with_scratch(const SeqHostArgs& h, void* scratch, size_t scratch_bytes,
                               cudaStream_t st);

}  // namespace externd
