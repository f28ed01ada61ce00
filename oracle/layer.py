"""fp64 oracle of the Gated DeltaNet-2 operator with the layer's processing
around it -- TEST INFRASTRUCTURE (only tests/, the smoke check and the
benchmark's CPU-baseline leg may use it).

"Gated DeltaNet-2", iplexlaw.co.kr, section "Procesamiento del token y
entrenamiento paralelo": queries and keys pass through a projection, a short
causal convolution, SiLU and L2 normalisation; values through a projection,
the convolution and SiLU; the recurrent output receives RMS normalisation, an
independent output gate (not the write gate) and a projection.  Section
"Decisiones independientes en dos ejes": the erase gate b and the write gate w
come from independent linear projections through sigmoid functions.

The projections, the convolution and the SiLU belong to the caller.  What sits
between them and the operator, and between the operator and the output
projection, is written out here in plain numpy, element by element and row by
row, in fp64:

    q_hat = q / sqrt(sum q^2 + EPS_L2)          (each token and head, over dk)
    k_hat = k / sqrt(sum k^2 + EPS_L2)
    b = sigmoid(b_logit),  w = sigmoid(w_logit)
    log_alpha = log(sigmoid(decay_logit))        (reading: alpha in (0, 1)
                                                  through the same sigmoid)
    o, S_T = operator(q_hat, k_hat, v, b, w, log_alpha, S0)    (oracle.fwd)
    y = o / sqrt(mean(o^2) + eps) * norm_weight * sigmoid(g_logit)
                                                 (each token and head, over dv;
                                                  reading: a sigmoid output gate)

The pages name neither the activation of the decay nor that of the output
gate, nor the epsilons; the readings above take the sigmoid the pages give for
the other gates, EPS_L2 = 1e-6, and the caller's eps for the RMS norm.
"""
from __future__ import annotations

import numpy as np

EPS_L2 = 1e-6


def _f64(x):
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def log_sigmoid(x):
    """log(1 / (1 + e^{-x})), written so that neither side overflows."""
    x = _f64(x)
    return np.minimum(x, 0.0) - np.log1p(np.exp(-np.abs(x)))


def sigmoid(x):
    """1 / (1 + e^{-x}), through its logarithm (no overflow for any x)."""
    return np.exp(log_sigmoid(x))


def l2_normalise(x):
    x = _f64(x)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + EPS_L2)


def prologue(q, k, b_logit, w_logit, decay_logit):
    """Normalised q and k, sigmoid gates and the log-decay."""
    return (l2_normalise(q), l2_normalise(k), sigmoid(b_logit), sigmoid(w_logit),
            log_sigmoid(decay_logit))


def epilogue(o, g_logit, norm_weight, eps):
    """RMS norm of each output row (over dv), times the weight and the output gate."""
    o = _f64(o)
    rms = np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + float(eps))
    return o / rms * _f64(norm_weight) * sigmoid(g_logit)


def layer_fwd(q, k, v, b_logit, w_logit, decay_logit, g_logit, norm_weight, eps, S0=None,
              nthreads: int = 0):
    """The operator with its prologue and epilogue; returns (y, S_T) in fp64."""
    import oracle
    qh, kh, b, w, la = prologue(q, k, b_logit, w_logit, decay_logit)
    o, st = oracle.fwd(qh, kh, _f64(v), b, w, la, S0=S0, nthreads=nthreads)
    return epilogue(o, g_logit, norm_weight, eps), st
