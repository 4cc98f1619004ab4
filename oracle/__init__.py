"""fp64 CPU oracle (test infrastructure; see ``apr_oracle``)."""
