"""Pure-Python brute force of the fused convolution, used only to pin the C
oracle on tiny shapes.  Python integers are unbounded and ``>>`` on a
negative int is a floor, so nothing here can overflow or truncate; it shares
no code with either the oracle or the CUDA path.

Definition (Inspur MLPerf ResNet50 convolution-merge article,
news.cnblogs.com/n/719672, sections 2.2 and 3.4: conv, then Bn, then the
shortcut Sum, then Relu, int8 out per section 3.1):
  t = (sum x*w + bias) * m + r * m_r + 2^(S-1);  out = clamp(t >> S, 0, 127)
"""


def brute_conv(x, w, bias, m, S, r=None, m_r=0):
    """x: nested lists [B][H][W][Ic]; w: [Oc][Ic][R][R]; r: [B][H][W][Oc] or None."""
    B, H, W, Ic = len(x), len(x[0]), len(x[0][0]), len(x[0][0][0])
    Oc, R = len(w), len(w[0][0])
    pad = (R - 1) // 2
    out = [[[[0] * Oc for _ in range(W)] for _ in range(H)] for _ in range(B)]
    for b in range(B):
        for h in range(H):
            for ww in range(W):
                for o in range(Oc):
                    acc = 0
                    for rr in range(R):
                        for ss in range(R):
                            hi, wi = h + rr - pad, ww + ss - pad
                            if 0 <= hi < H and 0 <= wi < W:
                                for i in range(Ic):
                                    acc += x[b][hi][wi][i] * w[o][i][rr][ss]
                    t = (acc + bias[o]) * m[o] + (r[b][h][ww][o] * m_r if r is not None else 0)
                    t += 1 << (S - 1)
                    out[b][h][ww][o] = min(max(t >> S, 0), 127)
    return out


def brute_conv_strided(x, w, bias, m, S, stride, pad, r=None, m_r=0):
    """Strided variant: output (b, ho, wo) reads input (ho*stride + rr - pad,
    wo*stride + ss - pad); output extent (n + 2*pad - R) // stride + 1."""
    B, H, W, Ic = len(x), len(x[0]), len(x[0][0]), len(x[0][0][0])
    Oc, R = len(w), len(w[0][0])
    Ho, Wo = (H + 2 * pad - R) // stride + 1, (W + 2 * pad - R) // stride + 1
    out = [[[[0] * Oc for _ in range(Wo)] for _ in range(Ho)] for _ in range(B)]
    for b in range(B):
        for ho in range(Ho):
            for wo in range(Wo):
                for o in range(Oc):
                    acc = 0
                    for rr in range(R):
                        for ss in range(R):
                            hi, wi = ho * stride + rr - pad, wo * stride + ss - pad
                            if 0 <= hi < H and 0 <= wi < W:
                                for i in range(Ic):
                                    acc += x[b][hi][wi][i] * w[o][i][rr][ss]
                    t = (acc + bias[o]) * m[o] + (r[b][ho][wo][o] * m_r if r is not None else 0)
                    t += 1 << (S - 1)
                    out[b][ho][wo][o] = min(max(t >> S, 0), 127)
    return out
