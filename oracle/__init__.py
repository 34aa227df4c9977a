"""Float64 CPU oracle of the gated delta rule -- test infrastructure only."""
