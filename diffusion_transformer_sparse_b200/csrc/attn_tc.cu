// Dispatch of the bf16 attention cores, all on the tensor cores: operands in
// tiled head layout (thl.cuh) go to the warp-specialised kernels of
// attn_rows_tc.cu (proxy self-attention, cross-attention, text
// cross-attention and full self-attention) and attn_win_tc.cu (window and
// shifted-window self-attention).
//
// Qihoo-T2X reading note, §3 Method: Eq. GIIM (SA among the proxies, CS with
// every latent the query and the proxies keys/values) and Eq. TCM (WSA, and
// SWSA on the grid rolled by -s with the wrapped pairs masked).
//
// The shapes they take: head widths 8 .. 80 in steps of 8 (one 64- or
// 80-column tile), and, for windows, 16, 32, 64 or 128 tokens (8, 4, 2 or 1
// windows per 128-row tile).  bf16 calls outside these shapes are refused by
// the API with PTDIT_ERR_SHAPE; there is no CUDA-core fallback for bf16.
#include "common.cuh"

namespace ptdit {

bool attention_thl_supported(const AttnArgs &a) {
    if (a.dtype != DT_BF16 || a.d < 8 || a.d > 80 || a.d % 8) return false;
    if (a.mode == ATT_WINDOW) {
        const int n = a.geom.n;
        return (n == 16 || n == 32 || n == 64 || n == 128) && a.q_bstride == a.k_bstride;
    }
    return a.nq >= 1 && a.nk >= 1;
}

bool attention_tc_supported(const AttnArgs &a) {
    return attention_thl_supported(a) && a.tq.mode != 0 && a.tk.mode != 0 && a.tv.mode != 0;
}

cudaError_t launch_attention_rows_tc(const AttnArgs &a, cudaStream_t s);
cudaError_t launch_attention_win_tc(const AttnArgs &a, cudaStream_t s);

cudaError_t launch_attention_tc(const AttnArgs &a, cudaStream_t s) {
    return a.mode == ATT_ROWS ? launch_attention_rows_tc(a, s) : launch_attention_win_tc(a, s);
}

}  // namespace ptdit
