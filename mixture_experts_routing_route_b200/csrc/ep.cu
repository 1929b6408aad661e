// Expert-parallel dispatch plans: which gathered rows go to which rank, and
// how a rank regroups the rows it receives into expert-major order for the
// grouped GEMM.
//
// Sources: "MoE Router: who decides which expert a token goes to" (the token
// dispatch: per-device send counts, device = expert / experts_per_device,
// then an all-to-all-v with per-pair counts and displacements; compute on
// the receiving device); "ops-transformer MoE operators" blog, 坑2 (tokens go
// to the cards that hold their experts and come back after the compute);
// "Integrating MoE into your model with Colossal-AI", step 2 (EP: all-to-all
// to the GPU holding the expert, expert MLP, all-to-all back).
//
// Experts are owned in contiguous blocks: rank g holds experts
// [g * E_loc, (g + 1) * E_loc). The permute already sorts the kept slots by
// expert, so the rows bound for rank g are one contiguous range of x_perm:
// the send plan is a scan over the kept counts. On the receiving side the
// rows arrive source-major (source 0's rows for this rank's experts, in
// expert order, then source 1's ...); the receive plan builds the
// expert-major order (for local expert e: source 0's rows, then source 1's)
// as a row map in both directions. The exchanges themselves are the
// caller's (NCCL all-to-all-v through torch.distributed in the binding).
#include "common.cuh"

namespace moe {
namespace {

constexpr int kEpThreads = 1024;

// send_rows[g] = sum of kept[e] over g's experts; send_offsets[g] = the first
// x_perm row for rank g (seg[g * E_loc]); send_offsets[world] = seg[E].
__global__ void __launch_bounds__(32) ep_send_plan_kernel(const int32_t* __restrict__ kept,
                                                          const int32_t* __restrict__ seg, int world,
                                                          int e_loc, int32_t* __restrict__ send_rows,
                                                          int32_t* __restrict__ send_offsets,
                                                          Control* ctl) {
  pdl_begin();
  for (int g = threadIdx.x; g < world; g += 32) {
    int n = 0;
    for (int i = 0; i < e_loc; ++i) {
      const int c = __ldg(kept + g * e_loc + i);
      if (c < 0) set_error(ctl, MOE_DEVERR_ROW_RANGE);
      n += max(c, 0);
    }
    send_rows[g] = n;
    send_offsets[g] = __ldg(seg + g * e_loc);
  }
  if (threadIdx.x == 0) send_offsets[world] = __ldg(seg + world * e_loc);
}

// counts: [world][e_loc] rows this rank receives from each source, per local
// expert (each source's kept counts for this rank's experts). One CTA:
//   recv_rows[s] = sum_e counts[s][e]; recv_offsets = exclusive scan;
//   local_seg[e] = exclusive scan over e of sum_s counts[s][e];
//   for local row r of expert e from source s (the i-th of that pair):
//     local_to_recv[r] = recv_offsets[s] + sum_{e' < e} counts[s][e'] + i,
//     recv_to_local[local_to_recv[r]] = r.
// A total above rows_cap is reported (MOE_DEVERR_ROW_RANGE) and no map is
// written.
__global__ void __launch_bounds__(kEpThreads) ep_recv_plan_kernel(
    const int32_t* __restrict__ counts, int world, int e_loc, long long rows_cap,
    int32_t* __restrict__ recv_rows, int32_t* __restrict__ recv_offsets,
    int32_t* __restrict__ local_seg, int32_t* __restrict__ local_to_recv,
    int32_t* __restrict__ recv_to_local, Control* ctl) {
  pdl_begin();
  extern __shared__ int32_t sh[];
  int32_t* c = sh;                            // [world][e_loc]
  int32_t* src_start = c + world * e_loc;     // [world][e_loc]: first recv row of (s, e)
  int32_t* pair_start = src_start + world * e_loc;  // [e_loc][world]: first local row of (s, e)
  __shared__ int bad_s;
  const int n = world * e_loc;
  if (threadIdx.x == 0) bad_s = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += kEpThreads) {
    const int v = __ldg(counts + i);
    if (v < 0) bad_s = 1;
    c[i] = max(v, 0);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // Sequential scans over world * e_loc <= 256 entries.
    long long off = 0;
    for (int s = 0; s < world; ++s) {
      recv_offsets[s] = static_cast<int32_t>(off);
      long long rs = 0;
      for (int e = 0; e < e_loc; ++e) {
        src_start[s * e_loc + e] = static_cast<int32_t>(off + rs);
        rs += c[s * e_loc + e];
      }
      recv_rows[s] = static_cast<int32_t>(rs);
      off += rs;
    }
    long long loc = 0;
    for (int e = 0; e < e_loc; ++e) {
      local_seg[e] = static_cast<int32_t>(loc);
      for (int s = 0; s < world; ++s) {
        pair_start[e * world + s] = static_cast<int32_t>(loc);
        loc += c[s * e_loc + e];
      }
    }
    local_seg[e_loc] = static_cast<int32_t>(loc);
    recv_offsets[world] = static_cast<int32_t>(off);
    if (bad_s || off > rows_cap || off >= 0x7fffffffLL) bad_s = 1;
  }
  __syncthreads();
  if (bad_s) {
    if (threadIdx.x == 0) set_error(ctl, MOE_DEVERR_ROW_RANGE);
    return;
  }
  // One warp per (source, expert) pair, its rows strided over the lanes.
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int p = warp; p < n; p += kEpThreads / 32) {
    const int s = p / e_loc, e = p - s * e_loc;
    const int cnt = c[p];
    const int r0 = src_start[p];
    const int l0 = pair_start[e * world + s];
    for (int i = lane; i < cnt; i += 32) {
      local_to_recv[l0 + i] = r0 + i;
      recv_to_local[r0 + i] = l0 + i;
    }
  }
}

}  // namespace

cudaError_t launch_ep_send_plan(const int32_t* kept, const int32_t* seg, int world, int e_loc,
                                int32_t* send_rows, int32_t* send_offsets, Control* ctl,
                                cudaStream_t s) {
  return launch_pdl(ep_send_plan_kernel, dim3(1), dim3(32), 0, s, false, kept, seg, world, e_loc,
                    send_rows, send_offsets, ctl);
}

static size_t ep_recv_plan_smem(int world, int e_loc) {
  return static_cast<size_t>(3) * world * e_loc * sizeof(int32_t);
}

cudaError_t launch_ep_recv_plan(const int32_t* counts, int world, int e_loc, long long rows_cap,
                                int32_t* recv_rows, int32_t* recv_offsets, int32_t* local_seg,
                                int32_t* local_to_recv, int32_t* recv_to_local, Control* ctl,
                                cudaStream_t s) {
  const size_t smem = ep_recv_plan_smem(world, e_loc);
  return launch_pdl(ep_recv_plan_kernel, dim3(1), dim3(kEpThreads), smem, s, false, counts, world,
                    e_loc, rows_cap, recv_rows, recv_offsets, local_seg, local_to_recv,
                    recv_to_local, ctl);
}

}  // namespace moe
