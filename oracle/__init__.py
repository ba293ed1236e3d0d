"""fp64 CPU oracle for the Kalman Delta Network (KDN) layer.

THIS PACKAGE IS TEST INFRASTRUCTURE. It is the slow, plain, obviously-correct
definition that the CUDA library is checked against. Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline / reference legs of
``bench.py`` may import it. The product path (``kalman_filter_linear_b200``)
never imports it and never falls back to it.

Modules:
  kdn_ref       token-by-token Isotropic / Diagonal KDN, the variance (Mobius)
                recurrence, its fp64 tree scan, and one decode step
  exact_kalman  the dense (full-covariance) Kalman filter of the same
                linear-Gaussian model, used to validate ``kdn_ref``
  deltanet      the gated delta rule driven by given write strengths
  kla_ref       the information-form diagonal filter (KLA): Mobius precision
                recursion, affine mean recursion, precision-ratio gates
  kdn_grad      the reverse-mode (adjoint) gradient of the KDN forward

Sources (page titles as printed on the pages):
  [KDN-abs]  "Kalman Delta Networks: Uncertainty-aware Associative Memory",
             English abstract (chatpaper.ai / zerohour.day copies)
  [KDN-sum]  "Kalman Delta Networks: 不确定性感知的联想记忆" (ai-feeds.com),
             sections 问题 / 核心洞察 / 方法 / 实验 / 局限
  [KLA]      "Kalman Linear Attention: Parallel Bayesian Filtering For
             Efficient Language Modelling and State Tracking" (gist.science),
             技术摘要 / 方法论 §1-§3 (the filter in information form, the
             Mobius form of the precision recursion, precision-ratio gates)

Parity pins: every function here is pinned against something other than
itself -- ``tests/test_oracle_pins.py`` (brute-force Gaussian conditioning,
numerical KL minimisation, closed forms, Mobius algebra, the gated delta rule,
invariants), ``tests/test_kla_pins.py`` (scalar-chain conditioning, the
Diagonal KDN special cases, the precision fixed point) and
``tests/test_grad_pins.py`` (finite differences of the forward).  The one
"parity unpinned" item is agreement with the KDN paper's own equations, which
no page prints: the reading of the process noise
(p_prior = a^2 p + w) and of the isotropic information scale (kappa = 1/d_k)
are the plainest readings the pages support, not the paper's verified text.
"""
