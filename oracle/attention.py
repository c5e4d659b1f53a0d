"""Dense GQA decode attention from packed records (the plain definition).

TEST INFRASTRUCTURE ONLY (see the package docstring).

Pages: the Block-GTQ abstract (a serving path that attends straight from the
packed cache) and the blockgtq README (fused decode over the packed K3V3 cache, compared with fp16
FlashAttention-2).  What that path computes is ordinary decode attention
over the dequantised cache:

    k_hat[D_g] = (n_g / sqrt(d_g)) * Pi_g^T C_b[codes_g]     for each K group
    v_hat      = (n_V / sqrt(D))   * Pi_V^T C_bV[codes_V]
    out_h      = sum_t softmax_t(q_h . k_hat_t / sqrt(D)) v_hat_t

with n the stored fp16 norms, C the fp16 codebook and Pi the fp32 rotations,
all in float64.
Query head h of the KV group reads the same cache.  Nothing here uses the
rotated-domain shortcut of the GPU path; tests check that the two agree.
"""
import numpy as np

def dequantise_keys(codes, k_norms, groups, rotations, codebooks, head_dim):
    """k_hat [T, D] float64 from record-order codes [T, P].

    groups: [(width, dims)]; rotations/codebooks keyed by width.
    """
    codes = np.asarray(codes, dtype=np.int64)
    t = codes.shape[0]
    k_hat = np.zeros((t, head_dim), dtype=np.float64)
    pos = 0
    for gi, (b, dims) in enumerate(groups):
        d = len(dims)
        c = codebooks[b].astype(np.float64)[codes[:, pos:pos + d]]          # [T, d]
        n = np.asarray(k_norms, dtype=np.float16)[:, gi].astype(np.float64)
        # row form of Pi^T c: c @ Pi
        k_hat[:, dims] = (n / np.sqrt(float(d)))[:, None] * (c @ rotations[b].astype(np.float64))
        pos += d
    return k_hat


def dequantise_values(codes, v_norms, rotation, codebook, head_dim):
    """v_hat [T, D] float64 for the single uniform V group from codes [T, D]."""
    c = codebook.astype(np.float64)[np.asarray(codes, dtype=np.int64)]
    n = np.asarray(v_norms, dtype=np.float16).astype(np.float64)
    return (n / np.sqrt(float(head_dim)))[:, None] * (c @ rotation.astype(np.float64))


def attend(q, k_hat, v_hat):
    """softmax(q k_hat^T / sqrt(D)) v_hat for q [G, D] float64; T = 0 gives zeros."""
    q = np.asarray(q, dtype=np.float64)
    if k_hat.shape[0] == 0:
        return np.zeros_like(q)
    logits = q @ k_hat.T / np.sqrt(float(q.shape[1]))
    logits -= logits.max(axis=1, keepdims=True)
    p = np.exp(logits)
    p /= p.sum(axis=1, keepdims=True)
    return p @ v_hat
