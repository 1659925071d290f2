"""CPU oracle (test infrastructure only; never imported by the CUDA path): ``zkv_oracle``
(numpy, float64) and its plain C twin ``zkv_oracle_c.c`` (wrapped by ``c_oracle``)."""
