// Arguments of the persistent decode kernel (internal to the library).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace ms {

// One layer as the persistent kernel sees it.  w[i]: tile-packed copy of matrix i (QKV, O,
// FC1, FC2): records of 16 rows x 32 columns, tile by tile (see launch_repack_tiles).
struct PLayer {
  const float *ln1_g, *ln1_b, *ln2_g, *ln2_b;
  const uint8_t* w[4];
};

struct PersistArgs {
  int L, d, H, Hk, F, V, fmt;
  float eps;
  const float* tok_emb;
  const float* lm_head;
  const float* lnf_g;
  const float* lnf_b;
  const PLayer* layers;      // device array [L]
  int cap;
  void* kc;                  // K cache base; layer l at element l * layer_stride
  void* vc;
  size_t layer_stride;       // elements
  int kv16;                  // cache elements are IEEE halves (else fp32)
  const float* cosv;         // RoPE table [cap][32]
  const float* sinv;
  int* dlen;                 // cache length (device)
  int32_t* hist;             // token history [cap][B]: argmax of position p at p * B + b
  unsigned* status;
  // Activation vectors handed from phase to phase as {value, epoch} 64-bit words.  vs[i]:
  // the outputs of matrix i (QKV, O, FC1, FC2) as up to 4 slices of [B][N_i] (each a
  // partial sum over a K range), vstride[i] words apart.
  uint64_t* vs[4];
  long long vstride[4];
  uint64_t* o_s;             // attention output [B][H * 64]
  unsigned epoch_base;       // epochs of this launch: epoch_base + 1 ...
  uint64_t* part_s;          // attention partials, stamped [B][Hk][att_splits][hpg][66]: m, l, o[64]
  int att_splits;
  float* lm_val;             // [grid][64]
  int* lm_idx;
  unsigned* lm_counter;
  unsigned* bar_count;       // grid barrier: arrivals, completed epoch, abort word
  unsigned* bar_flag;
  unsigned* abort;
  const int32_t* tokens_in;  // tokens of the first step [B], or null: take hist[(len - 1) * B + b]
  float* logits;             // [B][V] written every step, or null
  int32_t* argmax_out;       // [B] last step's argmax, or null
  int n_steps;
  int nslot;
  int sched_cap;             // capacity of the per-CTA slice table (entries)
  float guidance;            // 0, or classifier-free guidance over stream pairs (2p, 2p+1)
  long long settle_limit;    // rounds a stamped-word wait may take before it gives up
  long long grid_limit;      // polls of the grid barrier before it gives up
  int test_stall;            // tests only: 1 = an attention unit waits for a stamp no phase writes,
                             // 2 = the grid barrier waits for one arrival more than the grid makes
};
// Default wait limits (far above any legitimate wait, far below a hang).
constexpr long long kDefaultSettleLimit = 1ll << 23;
constexpr long long kDefaultGridLimit = 1ll << 24;

cudaError_t init_attrs_persistent();
// Ring slots that fit next to the kernel's other shared memory (0: the kernel does not fit).
int persistent_slots(int M, int L, int d, int H, int Hk, int F, int V, int G, int fmt, size_t smem_optin);
size_t persistent_smem(int M, int L, int d, int H, int Hk, int F, int V, int G, int fmt, int nslot);
// Upper bound on a CTA's weight slices per decode step (the slice table's entries).
int persistent_sched_cap(int L, int d, int H, int Hk, int F, int V, int G, int fmt);
// Whether the model's shapes suit the kernel for M streams on G CTAs (tiles per CTA,
// vector lengths); why gets a reason when not.
bool persistent_shapes_ok(int M, int d, int H, int Hk, int F, int V, int G, const char** why);
int persistent_max_ctas(int M, int fmt, size_t smem);
size_t persistent_static_smem(int M, int fmt);  // (size_t)-1 on error
cudaError_t launch_decode_persistent(const PersistArgs& a, int M, int grid, size_t smem, cudaStream_t st);

}  // namespace ms
